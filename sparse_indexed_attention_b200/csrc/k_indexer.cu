// Lightweight-indexer scores ([P2] "Hybrid Attention LLM Inference
// Acceleration...", section 2 item 2 and section 4(1); [P4] "Optimizing
// Inference for Hybrid-Architecture Large Language Models...", section 3.1):
//   score[t,s] = kI_scale[s] * sum_h w'[t,h] * ReLU(q^[t,h,:] . k^[s,:])
// read straight from the paged index cache; the head reduction happens in
// registers, so no [T, H_I, N] tensor is ever written.
//
// Simple CUDA-core form: one thread per candidate key, the token's 64 x 128
// query held in shared memory as fp32.
#include <cuda_fp8.h>

#include "dsa_internal.cuh"

namespace dsa {

namespace {

constexpr int kKeysPerBlock = 128;

template <bool kFp8>
__global__ void __launch_bounds__(kKeysPerBlock)
k_index_scores_simple(SeqsDev s, TokenMap tm, const void* __restrict__ q_operand,
                      const float* __restrict__ w_operand, const void* __restrict__ kI,
                      const float* __restrict__ kI_scale, float* __restrict__ scores, int64_t ld,
                      uint32_t* err) {
  const int t = blockIdx.x;
  const int pos = tm.pos[t];
  const int s0 = blockIdx.y * kKeysPerBlock;
  if (pos < 0 || s0 > pos) return;
  const int b = tm.seq[t];

  __shared__ float qs[kHI][kDI];
  __shared__ float ws[kHI];
  for (int i = threadIdx.x; i < kHI * kDI; i += blockDim.x) {
    float v;
    if constexpr (kFp8) {
      __nv_fp8_e4m3 c;
      c.__x = reinterpret_cast<const uint8_t*>(q_operand)[(int64_t)t * kHI * kDI + i];
      v = float(c);
    } else {
      v = __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(q_operand)[(int64_t)t * kHI * kDI + i]);
    }
    qs[i / kDI][i % kDI] = v;
  }
  if (threadIdx.x < kHI) ws[threadIdx.x] = w_operand[(int64_t)t * kHI + threadIdx.x];
  __syncthreads();

  const int sidx = s0 + threadIdx.x;
  if (sidx > pos) return;
  const int64_t row = phys_row(s.page_table, s.max_pages, s.num_phys_pages, b, sidx, err);
  if (row < 0) return;

  float k[kDI];
  if constexpr (kFp8) {
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const uint8_t*>(kI) + row * kDI);
#pragma unroll
    for (int c = 0; c < kDI / 16; ++c) {
      uint4 v = __ldg(src + c);
      const uint8_t* bytes = reinterpret_cast<const uint8_t*>(&v);
#pragma unroll
      for (int j = 0; j < 16; ++j) {
        __nv_fp8_e4m3 e;
        e.__x = bytes[j];
        k[c * 16 + j] = float(e);
      }
    }
  } else {
    const uint4* src = reinterpret_cast<const uint4*>(reinterpret_cast<const __nv_bfloat16*>(kI) + row * kDI);
#pragma unroll
    for (int c = 0; c < kDI / 8; ++c) {
      uint4 v = __ldg(src + c);
      const __nv_bfloat16* h = reinterpret_cast<const __nv_bfloat16*>(&v);
#pragma unroll
      for (int j = 0; j < 8; ++j) k[c * 8 + j] = __bfloat162float(h[j]);
    }
  }
  float acc = 0.f;
  for (int h = 0; h < kHI; ++h) {
    float d = 0.f;
#pragma unroll
    for (int i = 0; i < kDI; ++i) d = fmaf(qs[h][i], k[i], d);
    acc = fmaf(ws[h], fmaxf(d, 0.f), acc);
  }
  if constexpr (kFp8) acc *= __ldg(kI_scale + row);
  scores[(int64_t)t * ld + sidx] = acc;
}

}  // namespace

cudaError_t launch_index_scores(const SeqsDev& s, TokenMap tm, const void* q_operand, const float* w_operand,
                                const void* kI, const float* kI_scale, bool fp8, float* scores, int64_t ld,
                                uint32_t* err, cudaStream_t st) {
  dim3 grid(s.num_tokens, (s.max_ctx + kKeysPerBlock - 1) / kKeysPerBlock);
  if (fp8)
    k_index_scores_simple<true><<<grid, kKeysPerBlock, 0, st>>>(s, tm, q_operand, w_operand, kI, kI_scale,
                                                                 scores, ld, err);
  else
    k_index_scores_simple<false><<<grid, kKeysPerBlock, 0, st>>>(s, tm, q_operand, w_operand, kI, kI_scale,
                                                                  scores, ld, err);
  return counted(cudaGetLastError());
}

}  // namespace dsa
