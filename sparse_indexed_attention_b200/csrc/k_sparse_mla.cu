// Sparse MLA attention over the selected latent rows ([P1] "Day 0 Inference
// Adaptation and Performance Optimization for Hybrid Attention LLMs",
// Understanding the New Architecture item 2; [P2] "Hybrid Attention LLM
// Inference Acceleration...", section 2 item 2 "Sparse attention computation";
// [P5] "Day-0 Inference Adaptation for Large Language Models...", Operator
// Fusion and Memory Access Optimization, bullet 1: the Top-K indices go
// straight into the compute kernel, which gathers the rows itself).
//
//   out[t,h,:] = sum_{s in idx[t]} p_s KV[s,0:512],
//   p = softmax_s(scale * q[t,h,:] . KV[s,0:576]),   lse = ln sum exp(...)
//
// Simple CUDA-core form: a CTA owns (token, 16 heads, a slice of the index
// list), gathers 64 selected rows at a time into shared memory, and keeps an
// online softmax; slices of one token are merged by k_combine.
#include "dsa_internal.cuh"

namespace dsa {

namespace {

constexpr int kHG = 16;          // heads per CTA
constexpr int kChunk = 64;       // selected rows per shared-memory chunk
constexpr int kThreads = 256;
constexpr int kRowPad = kDQK + 8;  // bf16 elements per staged row (bank spread)

struct SmemLayout {
  float q[kHG][kDQK];
  __nv_bfloat16 kv[kChunk][kRowPad];
  float p[kHG][kChunk];
  float alpha[kHG];
  float m[kHG];
  float l[kHG];
  int64_t row[kChunk];
};

__device__ __forceinline__ void store_out(void* out, bool f32, int64_t i, float v) {
  if (f32)
    reinterpret_cast<float*>(out)[i] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16(v);
}

int attn_splits(int T, int H, int K) {
  int ctas = T * (H / kHG);
  int splits = 1;
  if (ctas < 2 * 148) {
    int want = (2 * 148 + ctas - 1) / ctas;
    int most = (K + kChunk - 1) / kChunk;
    splits = want < most ? want : most;
  }
  return splits;
}

int keys_per_split(int K, int splits) {
  int ks = (K + splits - 1) / splits;
  return (ks + kChunk - 1) / kChunk * kChunk;
}

__global__ void __launch_bounds__(kThreads)
k_sparse_mla_simple(SeqsDev s, TokenMap tm, const __nv_bfloat16* __restrict__ q,
                    const __nv_bfloat16* __restrict__ kv, const int32_t* __restrict__ idx, int K, int H,
                    float scale, int ks, int splits, void* __restrict__ out, bool out_f32, float* __restrict__ lse,
                    float* __restrict__ part_o, float2* __restrict__ part_ml, uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SmemLayout& sm = *reinterpret_cast<SmemLayout*>(smem_raw);
  const int t = blockIdx.x, hg = blockIdx.y, sp = blockIdx.z;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int pos = tm.pos[t];
  if (pos < 0) return;
  const int b = tm.seq[t];
  const int k_begin = sp * ks;
  const int k_end = min(K, k_begin + ks);

  for (int i = tid; i < kHG * kDQK; i += kThreads)
    sm.q[i / kDQK][i % kDQK] =
        __bfloat162float(q[((int64_t)t * H + hg * kHG + i / kDQK) * kDQK + i % kDQK]);
  if (tid < kHG) {
    sm.m[tid] = -INFINITY;
    sm.l[tid] = 0.f;
  }
  float acc[kHG][2];
#pragma unroll
  for (int h = 0; h < kHG; ++h) acc[h][0] = acc[h][1] = 0.f;

  for (int c0 = k_begin; c0 < k_end; c0 += kChunk) {
    __syncthreads();
    if (tid < kChunk) {
      int64_t r = -1;
      if (c0 + tid < k_end) {
        const int sidx = idx[(int64_t)t * K + c0 + tid];
        if (sidx >= 0 && sidx <= pos)
          r = phys_row(s.page_table, s.max_pages, s.num_phys_pages, b, sidx, err);
        else if (sidx != -1)
          raise_error(err, kErrBadIndex);
      }
      sm.row[tid] = r;
    }
    __syncthreads();
    for (int i = tid; i < kChunk * (kDQK / 8); i += kThreads) {
      const int j = i / (kDQK / 8), c = i % (kDQK / 8);
      uint4 v = make_uint4(0, 0, 0, 0);
      if (sm.row[j] >= 0) v = __ldg(reinterpret_cast<const uint4*>(kv + sm.row[j] * kDQK) + c);
      *reinterpret_cast<uint4*>(&sm.kv[j][c * 8]) = v;
    }
    __syncthreads();
    {  // logits: thread -> key j, heads 4*(tid/64) .. +3
      const int j = tid % kChunk, h0 = (tid / kChunk) * 4;
      float d[4] = {0.f, 0.f, 0.f, 0.f};
      for (int c = 0; c < kDQK; c += 8) {
        const uint4 v = *reinterpret_cast<const uint4*>(&sm.kv[j][c]);
        const __nv_bfloat16* e = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const float kvv = __bfloat162float(e[u]);
#pragma unroll
          for (int hh = 0; hh < 4; ++hh) d[hh] = fmaf(sm.q[h0 + hh][c + u], kvv, d[hh]);
        }
      }
      const bool valid = sm.row[j] >= 0;
#pragma unroll
      for (int hh = 0; hh < 4; ++hh) sm.p[h0 + hh][j] = valid ? d[hh] * scale : -INFINITY;
    }
    __syncthreads();
    // online softmax: warp w updates heads 2w, 2w+1
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      const int h = warp * 2 + r;
      const float v0 = sm.p[h][lane], v1 = sm.p[h][lane + 32];
      float cm = fmaxf(v0, v1);
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) cm = fmaxf(cm, __shfl_xor_sync(0xffffffffu, cm, o));
      const float m_old = sm.m[h];
      const float m_new = fmaxf(m_old, cm);
      float p0 = 0.f, p1 = 0.f, alpha = 1.f;
      if (m_new != -INFINITY) {
        p0 = __expf(v0 - m_new);
        p1 = __expf(v1 - m_new);
        alpha = __expf(m_old - m_new);
      }
      float ps = p0 + p1;
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) ps += __shfl_xor_sync(0xffffffffu, ps, o);
      __syncwarp();
      sm.p[h][lane] = p0;
      sm.p[h][lane + 32] = p1;
      if (lane == 0) {
        sm.alpha[h] = alpha;
        sm.m[h] = m_new;
        sm.l[h] = sm.l[h] * alpha + ps;
      }
    }
    __syncthreads();
    // O += p V : thread owns value dims tid and tid + 256 for all 16 heads
#pragma unroll
    for (int h = 0; h < kHG; ++h) {
      acc[h][0] *= sm.alpha[h];
      acc[h][1] *= sm.alpha[h];
    }
    for (int j = 0; j < kChunk; ++j) {
      const float v0 = __bfloat162float(sm.kv[j][tid]);
      const float v1 = __bfloat162float(sm.kv[j][tid + 256]);
#pragma unroll
      for (int h = 0; h < kHG; ++h) {
        const float p = sm.p[h][j];
        acc[h][0] = fmaf(p, v0, acc[h][0]);
        acc[h][1] = fmaf(p, v1, acc[h][1]);
      }
    }
  }
  __syncthreads();
  if (splits == 1) {
#pragma unroll
    for (int h = 0; h < kHG; ++h) {
      const float l = sm.l[h];
      const float inv = l > 0.f ? 1.f / l : 0.f;
      const int64_t o = ((int64_t)t * H + hg * kHG + h) * kDV;
      store_out(out, out_f32, o + tid, acc[h][0] * inv);
      store_out(out, out_f32, o + tid + 256, acc[h][1] * inv);
    }
    if (lse && tid < kHG) lse[(int64_t)t * H + hg * kHG + tid] = sm.m[tid] + logf(sm.l[tid]);
  } else {
#pragma unroll
    for (int h = 0; h < kHG; ++h) {
      const int64_t o = (((int64_t)t * splits + sp) * H + hg * kHG + h) * kDV;
      part_o[o + tid] = acc[h][0];
      part_o[o + tid + 256] = acc[h][1];
    }
    if (tid < kHG) part_ml[((int64_t)t * splits + sp) * H + hg * kHG + tid] = make_float2(sm.m[tid], sm.l[tid]);
  }
}

// Merge the split partials of one (token, head): rescale to the common max.
__global__ void __launch_bounds__(128)
k_combine(int H, int splits, const float* __restrict__ part_o, const float2* __restrict__ part_ml,
          const int32_t* __restrict__ tok_pos, void* __restrict__ out, bool out_f32, float* __restrict__ lse) {
  const int t = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  if (tok_pos[t] < 0) return;
  float M = -INFINITY;
  for (int i = 0; i < splits; ++i) M = fmaxf(M, part_ml[((int64_t)t * splits + i) * H + h].x);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int i = 0; i < splits; ++i) {
    const float2 ml = part_ml[((int64_t)t * splits + i) * H + h];
    if (ml.y == 0.f) continue;
    const float f = __expf(ml.x - M);
    L += ml.y * f;
    const float4 v = *reinterpret_cast<const float4*>(part_o + (((int64_t)t * splits + i) * H + h) * kDV + tid * 4);
    o[0] += v.x * f;
    o[1] += v.y * f;
    o[2] += v.z * f;
    o[3] += v.w * f;
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int64_t base = ((int64_t)t * H + h) * kDV + tid * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) store_out(out, out_f32, base + i, o[i] * inv);
  if (lse && tid == 0) lse[(int64_t)t * H + h] = M + logf(L);
}

}  // namespace

size_t sparse_mla_partials_bytes(int T, int K, int H) {
  const int splits = attn_splits(T, H, K);
  if (splits == 1) return 0;
  return (size_t)T * splits * H * (kDV * sizeof(float) + sizeof(float2));
}

cudaError_t launch_sparse_mla(const SeqsDev& s, TokenMap tm, const __nv_bfloat16* q, const __nv_bfloat16* kv,
                              const int32_t* idx, int K, int H, float scale, void* out, bool out_f32,
                              float* lse, void* partials, uint32_t* err, cudaStream_t st) {
  const int T = s.num_tokens;
  int splits = attn_splits(T, H, K);
  const int ks = keys_per_split(K, splits);
  splits = (K + ks - 1) / ks;
  float* part_o = reinterpret_cast<float*>(partials);
  float2* part_ml = reinterpret_cast<float2*>(part_o + (size_t)T * splits * H * kDV);
  const size_t smem = sizeof(SmemLayout);
  cudaError_t e = cudaSuccess;
  static thread_local int attr_set_for = -1;  // set once per device and thread, outside any capture
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_set_for != dev) {
    e = cudaFuncSetAttribute(k_sparse_mla_simple, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    attr_set_for = dev;
  }
  dim3 grid(T, H / kHG, splits);
  k_sparse_mla_simple<<<grid, kThreads, smem, st>>>(s, tm, q, kv, idx, K, H, scale, ks, splits, out, out_f32, lse, part_o,
                                                     part_ml, err);
  e = counted(cudaGetLastError());
  if (e != cudaSuccess || splits == 1) return e;
  k_combine<<<dim3(T, H), 128, 0, st>>>(H, splits, part_o, part_ml, tm.pos, out, out_f32, lse);
  return counted(cudaGetLastError());
}

}  // namespace dsa
