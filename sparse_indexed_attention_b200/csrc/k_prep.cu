// Per-token geometry and index-query quantization.
//
// token_map: the sequence and absolute position of every query token
//   (pos = ctx_len[b] - q_len[b] + j), validated once so that later kernels can
//   trust it; a token of an invalid sequence gets pos = -1 and sets the error
//   bit.
// quantize_index_query: the "Q quantization" input-preparation step of the
//   indexer ([P2] "Hybrid Attention LLM Inference Acceleration...", section
//   4(2); [P3] "Inference Acceleration for a New Domestic LLM Architecture...",
//   section 3 `q_quantize`).  One power-of-two scale per (token, head) row,
//   folded into the head weight.
#include <cuda_fp8.h>

#include "dsa_internal.cuh"

namespace dsa {

__global__ void k_token_map(SeqsDev s, int32_t* __restrict__ tok_seq, int32_t* __restrict__ tok_pos,
                            uint32_t* err) {
  int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= s.num_tokens) return;
  // sequence b with q_seq_start[b] <= t < q_seq_start[b+1] (binary search)
  int lo = 0, hi = s.batch - 1;
  while (lo < hi) {
    int mid = (lo + hi + 1) >> 1;
    if (__ldg(s.q_seq_start + mid) <= t) lo = mid; else hi = mid - 1;
  }
  int b = lo;
  int start = __ldg(s.q_seq_start + b), end = __ldg(s.q_seq_start + b + 1);
  int ctx = __ldg(s.ctx_len + b);
  int q_len = end - start;
  int pos = ctx - q_len + (t - start);
  bool ok = (__ldg(s.q_seq_start) == 0) && t >= start && t < end && ctx >= 1 && ctx <= s.max_ctx &&
            q_len <= ctx && ((ctx + kPage - 1) / kPage) <= s.max_pages && pos >= 0;
  if (!ok) {
    raise_error(err, kErrBadIndex);
    pos = -1;
  }
  tok_seq[t] = b;
  tok_pos[t] = pos;
}

cudaError_t launch_token_map(const SeqsDev& s, int32_t* tok_seq, int32_t* tok_pos, uint32_t* err,
                             cudaStream_t st) {
  int threads = 256;
  int blocks = (s.num_tokens + threads - 1) / threads;
  k_token_map<<<blocks, threads, 0, st>>>(s, tok_seq, tok_pos, err);
  return counted(cudaGetLastError());
}

// One warp per (token, head) row of 128 bf16: lane l holds elements 4l..4l+3.
__global__ void k_quantize_index_query(const __nv_bfloat16* __restrict__ qI, const float* __restrict__ w,
                                       int rows, uint8_t* __restrict__ codes, float* __restrict__ w_scaled) {
  int warp = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  int lane = threadIdx.x & 31;
  if (warp >= rows) return;
  const uint2 raw = __ldg(reinterpret_cast<const uint2*>(qI + (int64_t)warp * kDI) + lane);
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
  // x * 2^-e is exact in double; the result lies within [-448, 448].
  float y[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) y[i] = (float)ldexp((double)x[i], -e);
  __nv_fp8x2_storage_t c01 = __nv_cvt_float2_to_fp8x2(make_float2(y[0], y[1]), __NV_SATFINITE, __NV_E4M3);
  __nv_fp8x2_storage_t c23 = __nv_cvt_float2_to_fp8x2(make_float2(y[2], y[3]), __NV_SATFINITE, __NV_E4M3);
  uint32_t packed = (uint32_t)c01 | ((uint32_t)c23 << 16);
  reinterpret_cast<uint32_t*>(codes + (int64_t)warp * kDI)[lane] = packed;
  if (lane == 0) w_scaled[warp] = (float)ldexp((double)__ldg(w + warp), e);
}

cudaError_t launch_quantize_index_query(const __nv_bfloat16* qI, const float* w, int T, uint8_t* codes,
                                        float* w_scaled, cudaStream_t st) {
  int rows = T * kHI;
  int threads = 256;
  int blocks = (rows * 32 + threads - 1) / threads;
  k_quantize_index_query<<<blocks, threads, 0, st>>>(qI, w, rows, codes, w_scaled);
  return counted(cudaGetLastError());
}

}  // namespace dsa
