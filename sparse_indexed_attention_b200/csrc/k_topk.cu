// Top-K selection ([P3] "Inference Acceleration for a New Domestic LLM
// Architecture...", section 3 `topk_select`; [P2] "Hybrid Attention LLM
// Inference Acceleration...", section 2 item 2).
//
// Per row: the min(K, n) positions with the largest scores, equal scores ->
// lower position, emitted in ascending position order, padded with -1.  No
// sort of the row is ever materialised.
//
// Scores map to order-preserving 32-bit keys (-0.0 folded to +0.0 first);
// the key is resolved as three digits of 11, 11 and 10 bits.
//   1. histogram of digit 1 (the top 11 bits; lanes of a warp that hit the
//      same bin add once) -> the bin b1 that holds the K-th largest key;
//   2. one ordered pass keeps every position whose digit 1 is >= b1 as a
//      (position, key) pair, in position order -- fewer than K of them lie
//      above b1, the rest are b1's members -- and histograms digit 2 of b1's
//      members -> b2;
//   3. a histogram of digit 3 over the members of (b1, b2) gives the exact
//      key tau of the K-th largest and r = how many tau-valued keys are taken
//      (the lowest positions);
//   4. one ordered pass over the kept pairs emits every key > tau and the
//      first r keys == tau, already in position order.
// Rows much longer than the number of rows get several CTAs per row: steps 1
// and 2 run over chunks of the row in one kernel, and in a second kernel
// every CTA of the row resolves steps 3 and 4 from the row's kept pairs and
// writes the selections of its own chunk.  Otherwise one CTA does a row.  A degenerate row that
// keeps more pairs than shared memory holds is resolved from global memory
// (several CTAs per row) or by four 8-bit radix passes over the row (one CTA).
#include "sm100.cuh"
#include "topk_select.cuh"

namespace dsa {

namespace {

using namespace topk;
using sm100::cp_async_8;
using sm100::cp_async_16;
using sm100::cp_async_wait_all;

constexpr int kHistBins = kTopkHistBins;  // digit 1: key bits 31..21
constexpr int kLowBits = kTopkLowBits;
constexpr int kRowThreads = 1024;
constexpr int kRowStage = 12288;          // kept pairs in shared memory, one-CTA path
constexpr int kChunkThreads = 512;
constexpr int kMaxChunks = 64;
constexpr int kSelStage = 8192;           // kept pairs in shared memory, selecting CTA
constexpr int kPerThread = 8;             // consecutive scores per thread per pass



__device__ __forceinline__ int row_length(const int32_t* row_len, const int32_t* tok_pos, int t, int64_t ld,
                                          uint32_t* err) {
  const int64_t n64 = row_len ? (int64_t)row_len[t] : (int64_t)tok_pos[t] + 1;
  if (row_len && err && (n64 < 0 || n64 > ld)) raise_error(err, kErrBadIndex);
  return (int)(n64 < 0 ? 0 : (n64 > ld ? ld : n64));
}

// Keys of positions s0 .. s0+7 (those < end; others 0) and the bit mask of
// the ones that exist.  s0 is a multiple of 8; `vec` says the row start is
// 16-byte aligned, so two float4 loads serve a full run.
__device__ __forceinline__ uint32_t load_keys8(const float* __restrict__ row, int s0, int end, bool vec,
                                               uint32_t (&keys)[kPerThread]) {
  if (vec && s0 + kPerThread <= end) {
    const float4 a = __ldcg(reinterpret_cast<const float4*>(row + s0));
    const float4 b = __ldcg(reinterpret_cast<const float4*>(row + s0 + 4));
    keys[0] = order_key(a.x); keys[1] = order_key(a.y); keys[2] = order_key(a.z); keys[3] = order_key(a.w);
    keys[4] = order_key(b.x); keys[5] = order_key(b.y); keys[6] = order_key(b.z); keys[7] = order_key(b.w);
    return 0xFFu;
  }
  uint32_t have = 0;
#pragma unroll
  for (int j = 0; j < kPerThread; ++j) {
    keys[j] = 0;
    if (s0 + j < end) {
      keys[j] = order_key(__ldcg(row + s0 + j));
      have |= 1u << j;
    }
  }
  return have;
}

// Steps 3 and 4 for a row whose kept pairs (digit 1 >= b1, position order)
// are get(0 .. L-1).  hist holds digit 2's histogram of b1's members on entry
// (kD2Bins words, reused for digit 3); need = K - (keys above b1).
template <class Get>
__device__ void resolve_row(Get get, int L, uint32_t b1, uint32_t need, int K, uint32_t* hist, uint32_t* buf,
                            uint32_t* s_bin, uint32_t* s_above, int32_t* out) {
  find_bin<kD2Bins>(hist, need, s_bin, s_above);
  const uint32_t pre22 = (b1 << 11) | *s_bin;
  need -= *s_above;
  __syncthreads();  // every thread has read the result before the histogram is reused
  for (int i = threadIdx.x; i < kD3Bins; i += blockDim.x) hist[i] = 0u;
  __syncthreads();
  for (int base = 0; base < L; base += 4 * blockDim.x) {
    uint32_t key[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // loads first, then the (rarely active) adds
      const int i = base + u * blockDim.x + threadIdx.x;
      key[u] = i < L ? (uint32_t)get(i).y : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * blockDim.x + threadIdx.x;
      hist_add(hist, key[u] & (kD3Bins - 1), i < L && (key[u] >> 10) == pre22);
    }
  }
  __syncthreads();
  find_bin<kD3Bins>(hist, need, s_bin, s_above);
  const uint32_t tau = (pre22 << 10) | *s_bin;
  const uint32_t r = need - *s_above;
  emit_selected(L, tau, r, K, get, out, buf);
}

// ---------------------------------------------------------------- fallback
// Four 8-bit radix passes over the whole row, then the ordered emission.
__device__ void topk_row_full_radix(const float* __restrict__ row, int n, int K, int32_t* __restrict__ out,
                                    uint32_t* hist, uint32_t* buf, uint32_t* s_bin, uint32_t* s_above) {
  uint32_t prefix = 0, mask = 0, need = (uint32_t)K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = threadIdx.x; i < 256; i += blockDim.x) hist[i] = 0;
    __syncthreads();
    for (int base = 0; base < n; base += blockDim.x) {
      const int s = base + threadIdx.x;
      uint32_t key = 0;
      bool act = false;
      if (s < n) {
        key = order_key(row[s]);
        act = (key & mask) == prefix;
      }
      hist_add(hist, (key >> shift) & 0xFFu, act);
    }
    __syncthreads();
    find_bin<256>(hist, need, s_bin, s_above);
    prefix |= *s_bin << shift;
    mask |= 0xFFu << shift;
    need -= *s_above;
    __syncthreads();
  }
  emit_selected(
      n, prefix, need, K, [&](int i) { return make_int2(i, (int)order_key(row[i])); }, out, buf);
}

// ---------------------------------------------------------------- one CTA per row
struct RowSmem {
  uint32_t hist[kHistBins];
  uint32_t hist2[kD2Bins];
  uint32_t buf[33];
  uint32_t bin, above;
  int2 kept[kRowStage];
};

__global__ void __launch_bounds__(kRowThreads)
k_topk_row(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
           const int32_t* __restrict__ tok_pos, int K, int32_t* __restrict__ idx, uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowSmem& sm = *reinterpret_cast<RowSmem*>(smem_raw);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) {
    sm.hist[i] = 0;
    sm.hist2[i] = 0;
  }
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x;
  const float* __restrict__ row = scores + (int64_t)t * ld;
  int32_t* __restrict__ out = idx + (int64_t)t * K;
  const int n = row_length(row_len, tok_pos, t, ld, err);
  if (n <= K) {
    for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  __syncthreads();
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  for (int base = 0; base < n; base += blockDim.x * kPerThread) {
    uint32_t keys[kPerThread];
    const uint32_t have = load_keys8(row, base + threadIdx.x * kPerThread, n, vec, keys);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) hist_add(sm.hist, keys[j] >> kLowBits, (have >> j) & 1u);
  }
  __syncthreads();
  find_bin<kHistBins>(sm.hist, (uint32_t)K, &sm.bin, &sm.above);
  const uint32_t b1 = sm.bin, above = sm.above;
  const uint32_t L = above + sm.hist[b1];
  if (L > (uint32_t)kRowStage) {  // degenerate distribution: exact radix over the whole row
    __syncthreads();
    topk_row_full_radix(row, n, K, out, sm.hist, sm.buf, &sm.bin, &sm.above);
    return;
  }
  // keep (position, key) for digit 1 >= b1, in position order; digit 2 of b1's members
  uint32_t run = 0;
  for (int base = 0; base < n; base += blockDim.x * kPerThread) {
    const int s0 = base + threadIdx.x * kPerThread;
    uint32_t keys[kPerThread];
    const uint32_t have = load_keys8(row, s0, n, vec, keys);
    uint32_t keep = 0;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) keep |= (uint32_t)(((have >> j) & 1u) && (keys[j] >> kLowBits) >= b1) << j;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j)
      hist_add(sm.hist2, digit2(keys[j]), (keep >> j & 1u) && (keys[j] >> kLowBits) == b1);
    uint32_t total;
    uint32_t p = run + block_scan((uint32_t)__popc(keep), sm.buf, &total);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j)
      if (keep >> j & 1u) {
        if (p < (uint32_t)kRowStage) sm.kept[p] = make_int2(s0 + j, (int)keys[j]);
        ++p;
      }
    run += total;
  }
  __syncthreads();
  resolve_row([&](int i) { return sm.kept[i]; }, (int)L, b1, (uint32_t)K - above, K, sm.hist2, sm.buf, &sm.bin,
              &sm.above, out);
}

// ---------------------------------------------------------------- several CTAs per row
// Several CTAs per row: k_topk_hist (unless the indexer built the digit-1
// histogram), k_topk_filter, k_topk_emit; their scratch is laid out by
// launch_topk below.

__global__ void __launch_bounds__(kChunkThreads)
k_topk_hist(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
            const int32_t* __restrict__ tok_pos, int K, int chunk, uint32_t* __restrict__ ghist, uint32_t* err) {
  __shared__ uint32_t hist[kHistBins];
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y, c = blockIdx.x;
  const int n = row_length(row_len, tok_pos, t, ld, err);
  const int b0 = c * chunk, b1 = min(n, b0 + chunk);
  if (n <= K || b0 >= b1) return;
  __syncthreads();
  const float* __restrict__ row = scores + (int64_t)t * ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  for (int base = b0; base < b1; base += blockDim.x * kPerThread) {
    uint32_t keys[kPerThread];
    const uint32_t have = load_keys8(row, base + threadIdx.x * kPerThread, b1, vec, keys);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) hist_add(hist, keys[j] >> kLowBits, (have >> j) & 1u);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(&ghist[(int64_t)t * kHistBins + i], hist[i]);
}

struct FiltSmem {
  uint32_t hist[kHistBins];
  uint32_t hist2[kD2Bins];
  uint32_t buf[33];
  uint32_t bin, above;
};

// Steps 1-2 on chunk c of row t (digit-1 histogram already complete): the
// chunk's kept pairs, its share of the digit-2 histogram and its count;
// chunk 0 also records the row's b1 and the count of keys above it.
__global__ void __launch_bounds__(kChunkThreads)
k_topk_filter(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
              const int32_t* __restrict__ tok_pos, int K, int chunk, int C, const uint32_t* __restrict__ ghist,
              uint32_t* __restrict__ ghist2, int* __restrict__ counts, int2* __restrict__ kept,
              int2* __restrict__ row_info, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  FiltSmem& sm = *reinterpret_cast<FiltSmem*>(smem_raw);
  for (int i = threadIdx.x; i < kD2Bins; i += blockDim.x) sm.hist2[i] = 0;
  const int t = blockIdx.y, c = blockIdx.x;
  // row lengths come from the caller or from the call's first kernel, never
  // from the one just before: read them while it finishes
  const int n = row_length(row_len, tok_pos, t, ld, nullptr);
  pdl_wait();
  pdl_trigger();
  if (n <= K) {  // every candidate is selected
    int32_t* __restrict__ out = idx + (int64_t)t * K;
    if (c == 0)
      for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  const int b0 = c * chunk, b1 = min(n, b0 + chunk);
  for (int i = 4 * threadIdx.x; i < kHistBins; i += 4 * blockDim.x)
    cp_async_16(&sm.hist[i], ghist + (int64_t)t * kHistBins + i);
  // the first pass's scores are in flight together with the histogram
  const float* __restrict__ row = scores + (int64_t)t * ld;
  const bool vec = (reinterpret_cast<uintptr_t>(row) & 15) == 0;
  uint32_t keys[kPerThread];
  uint32_t have = load_keys8(row, b0 + threadIdx.x * kPerThread, b1, vec, keys);
  cp_async_wait_all();
  __syncthreads();
  find_bin<kHistBins>(sm.hist, (uint32_t)K, &sm.bin, &sm.above);
  const uint32_t bstar = sm.bin, above = sm.above;
  int2* my_kept = kept + ((int64_t)t * C + c) * chunk;
  uint32_t run = 0;
  for (int base = b0; base < b1; base += blockDim.x * kPerThread) {
    const int s0 = base + threadIdx.x * kPerThread;
    if (base != b0) have = load_keys8(row, s0, b1, vec, keys);
    uint32_t keep = 0;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j) keep |= (uint32_t)(((have >> j) & 1u) && (keys[j] >> kLowBits) >= bstar) << j;
#pragma unroll
    for (int j = 0; j < kPerThread; ++j)
      hist_add(sm.hist2, digit2(keys[j]), (keep >> j & 1u) && (keys[j] >> kLowBits) == bstar);
    uint32_t total;
    uint32_t p = run + block_scan((uint32_t)__popc(keep), sm.buf, &total);
#pragma unroll
    for (int j = 0; j < kPerThread; ++j)
      if (keep >> j & 1u) my_kept[p++] = make_int2(s0 + j, (int)keys[j]);  // p < chunk: one pair per position
    run += total;
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kD2Bins; i += blockDim.x)
    if (sm.hist2[i]) atomicAdd(&ghist2[(int64_t)t * kD2Bins + i], sm.hist2[i]);
  if (threadIdx.x == 0) {  // the next kernel reads these after this grid has completed
    counts[(int64_t)t * C + c] = (int)run;
    if (c == 0) row_info[t] = make_int2((int)bstar, (int)above);
  }
}

struct EmitSmem {
  uint32_t hist[kD2Bins];  // digit 2, then digit 3
  uint32_t buf[33];
  uint32_t bin, above;
  uint32_t before[2];      // earlier chunks' keys > tau and == tau
  int2 info;
  int off[kMaxChunks + 1];
  int2 kept[kSelStage];
};

// Steps 3-4 for row t: every CTA of the row resolves tau and r from the whole
// row's kept pairs (the same result in each), counts the earlier chunks'
// selections, and writes the selected positions of its own chunk c.
__global__ void __launch_bounds__(kChunkThreads)
k_topk_emit(int64_t ld, const int32_t* __restrict__ row_len, const int32_t* __restrict__ tok_pos, int K, int chunk,
            int C, const uint32_t* __restrict__ ghist2, const int* __restrict__ counts,
            const int2* __restrict__ kept, const int2* __restrict__ row_info, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  EmitSmem& sm = *reinterpret_cast<EmitSmem*>(smem_raw);
  const int t = blockIdx.y, c = blockIdx.x;
  const int n = row_length(row_len, tok_pos, t, ld, nullptr);  // not written by the kernel just before
  if (threadIdx.x < 2) sm.before[threadIdx.x] = 0u;
  pdl_wait();
  pdl_trigger();
  if (n <= K) return;  // written by the filter
  for (int i = 4 * threadIdx.x; i < kD2Bins; i += 4 * blockDim.x)
    cp_async_16(&sm.hist[i], ghist2 + (int64_t)t * kD2Bins + i);
  if (threadIdx.x < 32) {  // chunk counts -> offsets (two chunks per lane); the row's b1 / above
    const int lane = threadIdx.x;
    const int a0 = 2 * lane < C ? counts[(int64_t)t * C + 2 * lane] : 0;
    const int a1 = 2 * lane + 1 < C ? counts[(int64_t)t * C + 2 * lane + 1] : 0;
    int incl = a0 + a1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    sm.off[2 * lane] = incl - a0 - a1;
    sm.off[2 * lane + 1] = incl - a1;
    if (lane == 31) sm.off[kMaxChunks] = incl;
    if (lane == 0) sm.info = row_info[t];
  }
  __syncthreads();
  const int L = sm.off[C];  // offsets past C hold the same total
  const uint32_t b1 = (uint32_t)sm.info.x;
  uint32_t need = (uint32_t)K - (uint32_t)sm.info.y;
  const int2* row_kept = kept + (int64_t)t * C * chunk;
  const bool staged = L <= kSelStage;
  if (staged) {  // each warp copies whole chunks, every copy in flight at once
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, nw = blockDim.x >> 5;
    for (int cc = warp; cc < C; cc += nw) {
      const int o = sm.off[cc], cnt = sm.off[cc + 1] - o;
      for (int i = lane; i < cnt; i += 32) cp_async_8(&sm.kept[o + i], row_kept + (int64_t)cc * chunk + i);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  auto get = [&](int i) -> int2 {
    if (staged) return sm.kept[i];
    int lo = 0, hi = C - 1;  // degenerate row: last chunk whose offset <= i, read where it was left
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (sm.off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    return __ldcg(row_kept + (int64_t)lo * chunk + (i - sm.off[lo]));
  };
  // tau (the K-th largest key) and r (how many tau-valued keys are taken)
  find_bin<kD2Bins>(sm.hist, need, &sm.bin, &sm.above);
  const uint32_t pre22 = (b1 << 11) | sm.bin;
  need -= sm.above;
  __syncthreads();  // every thread has read the result before the histogram is reused
  for (int i = threadIdx.x; i < kD3Bins; i += blockDim.x) sm.hist[i] = 0u;
  __syncthreads();
  for (int base = 0; base < L; base += 4 * blockDim.x) {
    uint32_t key[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {  // loads first, then the (rarely active) adds
      const int i = base + u * blockDim.x + threadIdx.x;
      key[u] = i < L ? (uint32_t)get(i).y : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * blockDim.x + threadIdx.x;
      hist_add(sm.hist, key[u] & (kD3Bins - 1), i < L && (key[u] >> 10) == pre22);
    }
  }
  __syncthreads();
  find_bin<kD3Bins>(sm.hist, need, &sm.bin, &sm.above);
  const uint32_t tau = (pre22 << 10) | sm.bin;
  const uint32_t r = need - sm.above;
  // selections of the earlier chunks: pairs [0, off[c])
  const int o0 = sm.off[c], o1 = sm.off[c + 1];
  uint32_t gt = 0, eq = 0;
  for (int base = 0; base < o0; base += 4 * blockDim.x) {
    uint32_t key[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * blockDim.x + threadIdx.x;
      key[u] = i < o0 ? (uint32_t)get(i).y : 0u;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int i = base + u * blockDim.x + threadIdx.x;
      gt += (i < o0 && key[u] > tau) ? 1u : 0u;
      eq += (i < o0 && key[u] == tau) ? 1u : 0u;
    }
  }
  gt = __reduce_add_sync(0xffffffffu, gt);
  eq = __reduce_add_sync(0xffffffffu, eq);
  if ((threadIdx.x & 31) == 0) {
    atomicAdd(&sm.before[0], gt);
    atomicAdd(&sm.before[1], eq);
  }
  __syncthreads();
  const uint32_t eq_before = sm.before[1];
  const uint32_t taken_before = sm.before[0] + min(eq_before, r);
  const uint32_t r_left = r - min(eq_before, r);  // ties still to take, lowest positions first
  int32_t* __restrict__ out = idx + (int64_t)t * K + taken_before;
  emit_selected(
      o1 - o0, tau, r_left, K - (int)taken_before, [&](int i) { return get(o0 + i); }, out, sm.buf);
}

// Chunking of a row: several CTAs per row only when there are few rows.
void topk_chunks(int T, int64_t ld, int* C, int* chunk) {
  int c = 1;
  if (T < 2 * 148) {
    c = (2 * 148 + T - 1) / T;
    const int most = (int)((ld + 4095) / 4096);
    if (c > most) c = most;
    if (c > kMaxChunks) c = kMaxChunks;
    if (c < 1) c = 1;
  }
  int64_t ch = (ld + c - 1) / c;
  ch = (ch + 1023) / 1024 * 1024;
  *C = (int)((ld + ch - 1) / ch);
  *chunk = (int)ch;
}

template <class F>
cudaError_t set_smem_once(F* kernel, int bytes, int* dev_set) {
  int dev = 0;
  cudaGetDevice(&dev);
  if (*dev_set == dev) return cudaSuccess;
  cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  if (e == cudaSuccess) *dev_set = dev;
  return e;
}

int64_t pad16(int64_t x) { return (x + 15) / 16 * 16; }

}  // namespace

// Scratch layout (several CTAs per row): a region zeroed on every call --
// the per-row {b1, keys above b1} [T] (padded to 16 words), the digit-1
// histogram [T][2048] and the digit-2 histogram [T][2048] -- then counts
// [T][C] (padded to 16 words) and the kept pairs [T][C][chunk].
int64_t topk_zero_words(int T) { return pad16(2 * (int64_t)T) + (int64_t)T * (kHistBins + kD2Bins); }

size_t topk_scratch_bytes(int T, int64_t ld, int K) {
  (void)K;
  int C, chunk;
  topk_chunks(T, ld, &C, &chunk);
  if (C == 1) return 0;
  return (size_t)topk_zero_words(T) * 4 + (size_t)pad16((int64_t)T * C) * 4 + (size_t)T * C * chunk * sizeof(int2);
}

uint32_t* topk_hist_in_scratch(void* scratch, int T) {
  return reinterpret_cast<uint32_t*>(scratch) + pad16(2 * (int64_t)T);
}

bool topk_uses_hist(int T, int64_t ld) {
  int C, chunk;
  topk_chunks(T, ld, &C, &chunk);
  return C > 1;
}

cudaError_t launch_topk(const float* scores, int64_t ld, int T, const int32_t* row_len, const int32_t* tok_pos,
                        int K, int32_t* idx, void* scratch, bool hist_ready, uint32_t* err, cudaStream_t st) {
  int C, chunk;
  topk_chunks(T, ld, &C, &chunk);
  if (C == 1) {
    static thread_local int dev_row = -1;
    cudaError_t e = set_smem_once(k_topk_row, (int)sizeof(RowSmem), &dev_row);
    if (e != cudaSuccess) return e;
    e = launch_pdl("topk_row", k_topk_row, dim3(T), dim3(kRowThreads), sizeof(RowSmem), st, scores, ld, row_len,
                   tok_pos, K, idx, err);
    if (e != cudaSuccess) return e;
    return counted(cudaGetLastError());
  }
  int2* row_info = reinterpret_cast<int2*>(scratch);
  uint32_t* ghist = topk_hist_in_scratch(scratch, T);
  uint32_t* ghist2 = ghist + (int64_t)T * kHistBins;
  char* p = reinterpret_cast<char*>(scratch) + topk_zero_words(T) * 4;
  int* counts = reinterpret_cast<int*>(p);
  p += (size_t)pad16((int64_t)T * C) * 4;
  int2* kept = reinterpret_cast<int2*>(p);
  cudaError_t e = cudaSuccess;
  const dim3 grid(C, T);
  if (!hist_ready) {  // otherwise the caller has zeroed the region and filled the histogram
    if ((e = cudaMemsetAsync(scratch, 0, (size_t)topk_zero_words(T) * 4, st)) != cudaSuccess) return e;
    e = launch_pdl("topk_hist", k_topk_hist, grid, dim3(kChunkThreads), 0, st, scores, ld, row_len, tok_pos, K, chunk,
                   ghist, err);
    if (e != cudaSuccess || (e = counted(cudaGetLastError())) != cudaSuccess) return e;
  }
  static thread_local int dev_f = -1, dev_e = -1;
  if ((e = set_smem_once(k_topk_filter, (int)sizeof(FiltSmem), &dev_f)) != cudaSuccess) return e;
  if ((e = set_smem_once(k_topk_emit, (int)sizeof(EmitSmem), &dev_e)) != cudaSuccess) return e;
  e = launch_pdl("topk_filter", k_topk_filter, grid, dim3(kChunkThreads), sizeof(FiltSmem), st, scores, ld, row_len,
                 tok_pos, K, chunk, C, (const uint32_t*)ghist, ghist2, counts, kept, row_info, idx);
  if (e != cudaSuccess || (e = counted(cudaGetLastError())) != cudaSuccess) return e;
  e = launch_pdl("topk_emit", k_topk_emit, grid, dim3(kChunkThreads), sizeof(EmitSmem), st, ld, row_len, tok_pos, K,
                 chunk, C, (const uint32_t*)ghist2, (const int*)counts, (const int2*)kept, (const int2*)row_info,
                 idx);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace dsa
