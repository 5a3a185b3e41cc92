// Per-token geometry and index-query quantization.
//
// plan: the sequence and absolute position of every query token (pos =
//   ctx_len[b] - q_len[b] + j), validated once so that later kernels can trust
//   it, plus the indexer's work list (token groups x runs of key tiles), built
//   on the device so the host never needs the device-side lengths.
// quantize_index_query: the "Q quantization" input-preparation step of the
//   indexer ([P2] "Hybrid Attention LLM Inference Acceleration...", section
//   4(2); [P3] "Inference Acceleration for a New Domestic LLM Architecture...",
//   section 3 `q_quantize`).  For the E4M3 cache: one power-of-two scale per
//   (token, head) row, folded into the head weight.  For the MXFP8 cache
//   ([P2] section 5 table, "Indexer Q/K"; [P4] section 4.2): one E8M0 scale
//   per group of 32 elements, 2^(floor(log2 amax) - 8), kept as bytes
//   [T, 64, 4] for the indexer's block-scaled MMA.
#include <cuda_fp8.h>

#include "dsa_internal.cuh"

namespace dsa {

namespace {

__device__ __forceinline__ int warp_inclusive_scan(int v) {
  const int lane = threadIdx.x & 31;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += u;
  }
  return v;
}

// Exclusive prefix sum over a 1024-thread block; returns the thread's prefix
// and writes the block total to *total.
__device__ __forceinline__ int block_exclusive_scan(int v, int* warp_buf, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  int incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) warp_buf[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    const int w = warp_buf[lane];
    int wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    warp_buf[lane] = wi - w;
    if (lane == 31) warp_buf[32] = wi;
  }
  __syncthreads();
  const int r = warp_buf[warp] + incl - v;
  *total = warp_buf[32];
  __syncthreads();
  return r;
}

// Sequences whose q_seq_start / ctx_len the plan stages in shared memory
// (larger batches are read from global memory).
constexpr int kPlanSeqs = 1024;

// qs / cl: q_seq_start and ctx_len, staged in shared memory or global.
__device__ __forceinline__ bool seq_ok(const SeqsDev& s, const int* qs, const int* cl, int b, int* q_len_out,
                                       int* ctx_out) {
  const int q_len = qs[b + 1] - qs[b];
  const int ctx = cl[b];
  *q_len_out = q_len;
  *ctx_out = ctx;
  // the sequence's query rows lie inside the T rows of every per-token tensor
  return q_len >= 0 && qs[b] >= 0 && qs[b + 1] <= s.num_tokens && ctx >= 1 && ctx <= s.max_ctx && q_len <= ctx &&
         (ctx + kPage - 1) / kPage <= s.max_pages;
}

}  // namespace

// One CTA of 1024 threads.  Writes
//   tok_seq/tok_pos [T]   sequence and absolute position of every query token
//                         (pos = -1 and the error bit for an invalid one);
//   groups [G]            {b, t0, cnt, pos0}: up to `tg` consecutive query tokens
//                         of one sequence (their positions are pos0 .. pos0+cnt-1);
//   items [I]             two int4 per item: {b, t0, cnt, pos0} of its group and
//                         {tile_begin, tile_end, g, 0}: a run of <= `ch` key tiles
//                         of 128 positions (tiles cover 0 .. last pos);
//   counts                {G, I}.
// The plan's shared memory (declared once, used by either instantiation).
struct PlanSmem {
  int warp_buf[33];
  int qs[kPlanSeqs + 1], cl[kPlanSeqs], gs[kPlanSeqs + 1];  // staged sequence arrays
  int istart[1025];
  int tiles[1024];
  int4 gd[1024];
};

template <bool kStaged>
__device__ __forceinline__ void plan_impl(const SeqsDev& s, int tg, int ch, const PlanBufs& p, uint32_t* err,
                                          PlanSmem& sm) {
  int* warp_buf = sm.warp_buf;
  int* sh_qs = sm.qs;
  int* sh_cl = sm.cl;
  int* sh_gs = sm.gs;
  const int tid = threadIdx.x;
  // staged: one round of coalesced loads instead of chains of dependent ones
  if constexpr (kStaged) {
    for (int b = tid; b <= s.batch; b += blockDim.x) {
      sh_qs[b] = __ldg(s.q_seq_start + b);
      if (b < s.batch) sh_cl[b] = __ldg(s.ctx_len + b);
    }
    __syncthreads();
  }
  const int* qs = kStaged ? sh_qs : s.q_seq_start;
  const int* cl = kStaged ? sh_cl : s.ctx_len;
  int* gs = kStaged ? sh_gs : p.seq_gstart;
  for (int t = tid; t < s.num_tokens; t += blockDim.x) {
    int lo = 0, hi = s.batch - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (qs[mid] <= t) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int start = qs[b], end = qs[b + 1];
    int q_len, ctx;
    const bool ok = seq_ok(s, qs, cl, b, &q_len, &ctx) && qs[0] == 0 && t >= start && t < end;
    int pos = ctx - q_len + (t - start);
    if (!ok || pos < 0) {
      raise_error(err, kErrBadIndex);
      pos = -1;
    }
    p.tok_seq[t] = b;
    p.tok_pos[t] = pos;
  }
  if (ch <= 0) return;  // token geometry only
  // groups per sequence -> start offsets (an invalid sequence gets none)
  auto groups_of = [&](int b) -> int {
    int cnt = 0;
    if (b < s.batch) {
      int q_len, ctx;
      if (seq_ok(s, qs, cl, b, &q_len, &ctx))
        cnt = (q_len + tg - 1) / tg;
      else
        raise_error(err, kErrBadIndex);
    }
    return cnt;
  };
  int running = 0;
  if (s.batch <= 32) {  // one warp, shuffles only
    if (tid < 32) {
      const int cnt = groups_of(tid);
      const int incl = warp_inclusive_scan(cnt);
      if (tid < s.batch) {
        gs[tid] = incl - cnt;
        p.seq_gstart[tid] = incl - cnt;
      }
      if (tid == 31) {  // lanes past the batch add nothing
        gs[s.batch] = incl;
        p.seq_gstart[s.batch] = incl;
      }
    }
    __syncthreads();
    running = gs[s.batch];
  } else {
    for (int base = 0; base < s.batch; base += blockDim.x) {
      const int b = base + tid;
      const int cnt = groups_of(b);
      int total;
      const int excl = block_exclusive_scan(cnt, warp_buf, &total);
      if (b < s.batch) {
        gs[b] = running + excl;
        p.seq_gstart[b] = running + excl;
      }
      running += total;
    }
    if (tid == 0) {
      gs[s.batch] = running;
      p.seq_gstart[s.batch] = running;
    }
    __syncthreads();
  }
  const int G = running;
  // Sequences whose query rows do not overlap give at most plan_max_groups
  // groups, the capacity the workspace holds.  Only a q_seq_start that
  // decreases somewhere (overlapping rows) gives more: no work is planned and
  // the error is raised.
  if (G > plan_max_groups(s.num_tokens, s.batch, tg)) {
    if (tid == 0) {
      raise_error(err, kErrBadIndex);
      p.counts[0] = 0;
      p.counts[1] = 0;
    }
    return;
  }
  int* s_istart = sm.istart;
  int* s_tiles = sm.tiles;
  int4* s_gd = sm.gd;
  // group g: its descriptor, key tiles and work items
  auto describe = [&](int g, int* tiles, int* nitems) -> int4 {
    int lo = 0, hi = s.batch - 1;  // largest b with seq_gstart[b] <= g
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (gs[mid] <= g) lo = mid; else hi = mid - 1;
    }
    const int b = lo;
    const int q_len = qs[b + 1] - qs[b];
    const int j0 = (g - gs[b]) * tg;
    const int cnt = min(tg, q_len - j0);
    const int pos0 = cl[b] - q_len + j0;
    *tiles = (pos0 + cnt - 1) / 128 + 1;
    *nitems = (*tiles + ch - 1) / ch;
    return make_int4(b, qs[b] + j0, cnt, pos0);
  };
  // items [irun, irun + total) of groups gbase .. gbase + ng - 1, whose
  // prefixes / tiles / descriptors sit in s_istart / s_tiles / s_gd
  auto write_items = [&](int irun, int total, int gbase, int ng) {
    for (int i = tid; i < total; i += blockDim.x) {
      int lo = 0, hi = ng - 1;  // last local group with s_istart <= i
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (s_istart[mid] <= i) lo = mid; else hi = mid - 1;
      }
      const int j = i - s_istart[lo];
      const int tl = s_tiles[lo];
      p.items[2 * (irun + i)] = s_gd[lo];
      p.items[2 * (irun + i) + 1] = make_int4(j * ch, min(tl, (j + 1) * ch), gbase + lo, 0);
    }
  };
  int irun = 0;
  if (G <= 32) {  // one warp, shuffles only
    if (tid < 32) {
      int nitems = 0, tiles = 0;
      int4 gd = make_int4(0, 0, 0, 0);
      if (tid < G) {
        gd = describe(tid, &tiles, &nitems);
        p.groups[tid] = gd;
      }
      const int incl = warp_inclusive_scan(nitems);
      s_istart[tid] = incl - nitems;
      s_tiles[tid] = tiles;
      s_gd[tid] = gd;
      if (tid == 31) s_istart[32] = incl;
    }
    __syncthreads();
    irun = s_istart[32];
    write_items(0, irun, 0, G);
  } else {
    for (int gbase = 0; gbase < G; gbase += blockDim.x) {
      const int g = gbase + tid;
      int nitems = 0, tiles = 0;
      int4 gd = make_int4(0, 0, 0, 0);
      if (g < G) {
        gd = describe(g, &tiles, &nitems);
        p.groups[g] = gd;
      }
      int total;
      const int excl = block_exclusive_scan(nitems, warp_buf, &total);
      s_istart[tid] = excl;
      s_tiles[tid] = tiles;
      s_gd[tid] = gd;
      if (tid == 0) s_istart[blockDim.x] = total;
      __syncthreads();
      write_items(irun, total, gbase, min((int)blockDim.x, G - gbase));
      irun += total;
      __syncthreads();
    }
  }
  if (tid == 0) {
    p.counts[0] = G;
    p.counts[1] = irun;
  }
}

__device__ __forceinline__ void plan_body(const SeqsDev& s, int tg, int ch, const PlanBufs& p, uint32_t* err) {
  __shared__ PlanSmem sm;
  if (s.batch <= kPlanSeqs)
    plan_impl<true>(s, tg, ch, p, err, sm);
  else
    plan_impl<false>(s, tg, ch, p, err, sm);
}

__global__ void __launch_bounds__(1024) k_plan(SeqsDev s, int tg, int ch, PlanBufs p, uint32_t* err) {
  pdl_wait();
  pdl_trigger();
  plan_body(s, tg, ch, p, err);
}

cudaError_t launch_plan(const SeqsDev& s, int tg, int ch, const PlanBufs& p, uint32_t* err, cudaStream_t st) {
  cudaError_t e = launch_pdl("plan", k_plan, dim3(1), dim3(1024), 0, st, s, tg, ch, p, err);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

// One warp quantizes one (token, head) row of 128 bf16: lane l holds elements 4l..4l+3.
__device__ __forceinline__ void quant_row(const __nv_bfloat16* __restrict__ qI, const float* __restrict__ w, int row,
                                          uint8_t* __restrict__ codes, float* __restrict__ w_scaled) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qI + (int64_t)row * kDI) + lane);
  __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  float x[4] = {__low2float(p0), __high2float(p0), __low2float(p1), __high2float(p1)};
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));
  // e = smallest integer with amax <= 448 * 2^e; compared exactly (448 * 2^e is
  // representable for every e reachable from a finite bf16 amax).
  int e = 0;
  if (amax > 0.f) {
    int ex;
    frexpf(amax / 448.f, &ex);  // estimate, corrected below by exact comparisons
    e = ex;
    while (amax > ldexpf(448.f, e)) ++e;
    while (amax <= ldexpf(448.f, e - 1)) --e;
  }
  // x * 2^-e, correctly rounded (exact unless the result is subnormal, where
  // E4M3 rounds it to zero anyway); the result lies within [-448, 448].
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = ldexpf(x[i], -e);
  __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(make_float2(y[0], y[1]), __NV_SATFINITE, __NV_E4M3);
  __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(make_float2(y[2], y[3]), __NV_SATFINITE, __NV_E4M3);
  const uint32_t packed = (uint32_t)c01 | ((uint32_t)c23 << 16);
  reinterpret_cast<uint32_t*>(codes + (int64_t)row * kDI)[lane] = packed;
  if (lane == 0) w_scaled[row] = ldexpf(__ldg(w + row), e);
}

// MXFP8: one warp per (token, head) row of 128 bf16; lane l holds elements
// 4l..4l+3, so lanes 8g..8g+7 hold group g.  The group's shared exponent is
// floor(log2 amax) - 8 (from frexpf, exact for any finite float), clamped to
// [-127, 127]; an all-zero group takes 0.  Elements divided by 2^e (exact)
// round to E4M3 with saturation; the scale goes out as its E8M0 byte e + 127.
__device__ __forceinline__ void quant_row_mx(const __nv_bfloat16* __restrict__ qI, int row, uint8_t* __restrict__ codes,
                                             uint8_t* __restrict__ scales) {
  const int lane = threadIdx.x & 31;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qI + (int64_t)row * kDI) + lane);
  __nv_bfloat162 p0 = *reinterpret_cast<const __nv_bfloat162*>(&raw.x);
  __nv_bfloat162 p1 = *reinterpret_cast<const __nv_bfloat162*>(&raw.y);
  float x[4] = {__low2float(p0), __high2float(p0), __low2float(p1), __high2float(p1)};
  float amax = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
  for (int o = 4; o > 0; o >>= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, o));  // within the 8-lane group
  int e = 0;
  if (amax > 0.f) {
    int ex;
    frexpf(amax, &ex);  // amax = m * 2^ex, 0.5 <= m < 1
    e = min(127, max(-127, ex - 9));
  }
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = ldexpf(x[i], -e);
  __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(make_float2(y[0], y[1]), __NV_SATFINITE, __NV_E4M3);
  __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(make_float2(y[2], y[3]), __NV_SATFINITE, __NV_E4M3);
  reinterpret_cast<uint32_t*>(codes + (int64_t)row * kDI)[lane] = (uint32_t)c01 | ((uint32_t)c23 << 16);
  if ((lane & 7) == 0) scales[(int64_t)row * 4 + (lane >> 3)] = (uint8_t)(e + 127);
}

__global__ void k_quantize_index_query_mx(const __nv_bfloat16* __restrict__ qI, int rows, uint8_t* __restrict__ codes,
                                          uint8_t* __restrict__ scales) {
  pdl_wait();
  pdl_trigger();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row < rows) quant_row_mx(qI, row, codes, scales);
}

__global__ void k_quantize_index_query(const __nv_bfloat16* __restrict__ qI, const float* __restrict__ w,
                                       int rows, uint8_t* __restrict__ codes, float* __restrict__ w_scaled) {
  pdl_wait();
  pdl_trigger();
  const int row = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  if (row < rows) quant_row(qI, w, row, codes, w_scaled);
}

// Everything the indexer needs before it starts, in one launch: block 0 builds
// the plan; the other blocks quantize the index query (32 rows per block, FP8
// and MXFP8 caches only) and zero a scratch range (Top-K's first-digit
// histogram).
struct PrepArgs {
  SeqsDev s;
  int tg, ch;
  PlanBufs plan;
  uint32_t* err;
  const __nv_bfloat16* qI;
  const float* w;
  uint8_t* codes;
  float* w_scaled;
  uint8_t* q_sf;  // MXFP8: E8M0 group scales [rows, 4] (w_scaled unused)
  int quant_rows;
  uint32_t* zero;
  int64_t zero_words;
};

__global__ void __launch_bounds__(1024) k_prep(const PrepArgs a) {
  pdl_wait();  // the previous call may still read the plan and the scratch this kernel rewrites
  pdl_trigger();
  if (blockIdx.x == 0) {
    plan_body(a.s, a.tg, a.ch, a.plan, a.err);
    return;
  }
  const int b = blockIdx.x - 1, nb = gridDim.x - 1;
  if (a.qI) {
    const int row = b * 32 + (threadIdx.x >> 5);
    if (row < a.quant_rows) {
      if (a.q_sf)
        quant_row_mx(a.qI, row, a.codes, a.q_sf);
      else
        quant_row(a.qI, a.w, row, a.codes, a.w_scaled);
    }
  }
  if (a.zero) {
    const int64_t per = (a.zero_words + nb - 1) / nb;
    const int64_t z0 = (int64_t)b * per, z1 = min(a.zero_words, z0 + per);
    for (int64_t i = z0 + threadIdx.x; i < z1; i += blockDim.x) a.zero[i] = 0u;
  }
}

cudaError_t launch_prep(const SeqsDev& s, int tg, int ch, const PlanBufs& plan, const __nv_bfloat16* qI,
                        const float* w, uint8_t* codes, float* w_scaled, uint8_t* q_sf, uint32_t* zero,
                        int64_t zero_words, uint32_t* err, cudaStream_t st) {
  PrepArgs a{s,     tg,   ch, plan, err, qI, w, codes, w_scaled, q_sf, qI ? s.num_tokens * kHI : 0,
             zero, zero ? zero_words : 0};
  const int64_t nq = qI ? ((int64_t)s.num_tokens * kHI + 31) / 32 : 0;
  const int64_t nz = zero ? (zero_words + 4095) / 4096 : 0;
  const int64_t extra = nq > nz ? nq : nz;
  cudaError_t e = launch_pdl("prep", k_prep, dim3((unsigned)(1 + extra)), dim3(1024), 0, st, a);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

cudaError_t launch_quantize_index_query_mx(const __nv_bfloat16* qI, int T, uint8_t* codes, uint8_t* scales,
                                           cudaStream_t st) {
  const int rows = T * kHI, threads = 256;
  const int blocks = (rows * 32 + threads - 1) / threads;
  cudaError_t e = launch_pdl("quantize_index_query_mx", k_quantize_index_query_mx, dim3(blocks), dim3(threads), 0, st,
                             qI, rows, codes, scales);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

cudaError_t launch_quantize_index_query(const __nv_bfloat16* qI, const float* w, int T, uint8_t* codes,
                                        float* w_scaled, cudaStream_t st) {
  int rows = T * kHI;
  int threads = 256;
  int blocks = (rows * 32 + threads - 1) / threads;
  cudaError_t e = launch_pdl("quantize_index_query", k_quantize_index_query, dim3(blocks), dim3(threads), 0, st, qI, w, rows, codes, w_scaled);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace dsa
