// Top-K selection ([P3] "Inference Acceleration for a New Domestic LLM
// Architecture...", section 3 `topk_select`; [P2] "Hybrid Attention LLM
// Inference Acceleration...", section 2 item 2).
//
// Per row: the min(K, n) positions with the largest scores, equal scores ->
// lower position, emitted in ascending position order, padded with -1.  No
// sort is ever materialised:
//   1. scores map to order-preserving 32-bit keys (-0.0 first folded to +0.0);
//   2. a most-significant-digit radix select (four 8-bit digits, shared-memory
//      histograms) finds the exact key tau of the K-th largest score and how
//      many tau-valued positions, r, are taken (the r lowest ones);
//   3. one ordered pass emits every position with key > tau, and tau-valued
//      positions while fewer than r have been emitted, at offsets given by a
//      block-wide prefix sum -- so the output is ascending and exact.
#include "dsa_internal.cuh"

namespace dsa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;

__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;  // -0.0 ranks equal to +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__global__ void __launch_bounds__(kThreads)
k_topk_row(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
           const int32_t* __restrict__ tok_pos, int K, int32_t* __restrict__ idx, uint32_t* err) {
  const int t = blockIdx.x;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* __restrict__ row = scores + (int64_t)t * ld;
  int32_t* __restrict__ out = idx + (int64_t)t * K;

  int64_t n64 = row_len ? (int64_t)row_len[t] : (int64_t)tok_pos[t] + 1;
  if (row_len && (n64 < 0 || n64 > ld)) raise_error(err, kErrBadIndex);
  const int n = (int)(n64 < 0 ? 0 : (n64 > ld ? ld : n64));

  if (n <= K) {  // every candidate is selected
    for (int i = tid; i < K; i += kThreads) out[i] = i < n ? i : -1;
    return;
  }

  __shared__ uint32_t hist[256];
  __shared__ uint32_t s_digit, s_krem;
  __shared__ uint32_t warp_sums[kWarps];
  __shared__ uint32_t s_run_gt, s_run_eq;

  // ---- radix select: exact key of the K-th largest score ----
  uint32_t prefix = 0, mask = 0, krem = (uint32_t)K;
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    for (int i = tid; i < 256; i += kThreads) hist[i] = 0;
    __syncthreads();
    for (int s = tid; s < n; s += kThreads) {
      const uint32_t key = order_key(row[s]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 0xFFu], 1u);
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l down to 248-8l; scan from the top digit
      uint32_t c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[255 - 8 * lane - j];
        sum += c[j];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += v;
      }
      const uint32_t excl = incl - sum;  // keys (with this prefix) above the lane's digits
      if (excl < krem && krem <= incl) {
        uint32_t above = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + c[j] >= krem) {
            s_digit = 255u - 8u * lane - j;
            s_krem = krem - above;
            break;
          }
          above += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= s_digit << shift;
    mask |= 0xFFu << shift;
    krem = s_krem;
    __syncthreads();
  }
  const uint32_t tau = prefix;  // key of the K-th largest score
  // krem = number of tau-valued positions to take (the lowest ones)

  // ---- ordered emission ----
  if (tid == 0) {
    s_run_gt = 0;
    s_run_eq = 0;
  }
  __syncthreads();
  for (int base = 0; base < n; base += kThreads * 4) {
    const int s0 = base + tid * 4;
    uint32_t gt = 0, eq = 0;  // bit j: element s0+j is above / equal to tau
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (s0 + j < n) {
        const uint32_t key = order_key(row[s0 + j]);
        gt |= (key > tau) << j;
        eq |= (key == tau) << j;
      }
    }
    const uint32_t packed = ((uint32_t)__popc(gt) << 16) | (uint32_t)__popc(eq);
    uint32_t incl = packed;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t v = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += v;
    }
    if (lane == 31) warp_sums[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      const uint32_t v = warp_sums[lane];
      uint32_t wi = v;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, wi, o);
        if (lane >= o) wi += u;
      }
      warp_sums[lane] = wi - v;  // exclusive
    }
    __syncthreads();
    const uint32_t excl = warp_sums[warp] + incl - packed;
    const uint32_t run_gt = s_run_gt, run_eq = s_run_eq;
    uint32_t eq_before = run_eq + (excl & 0xFFFFu);
    uint32_t p = run_gt + (excl >> 16) + min(eq_before, krem);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (gt >> j & 1u) {
        if (p < (uint32_t)K) out[p] = s0 + j;  // p < K always holds; the guard keeps writes in bounds regardless
        ++p;
      } else if (eq >> j & 1u) {
        if (eq_before < krem) {
          if (p < (uint32_t)K) out[p] = s0 + j;
          ++p;
        }
        ++eq_before;
      }
    }
    __syncthreads();
    if (tid == kThreads - 1) {
      const uint32_t total = excl + packed;
      s_run_gt = run_gt + (total >> 16);
      s_run_eq = run_eq + (total & 0xFFFFu);
    }
    __syncthreads();
  }
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, int T, const int32_t* row_len, const int32_t* tok_pos,
                        int K, int32_t* idx, uint32_t* err, cudaStream_t st) {
  k_topk_row<<<T, kThreads, 0, st>>>(scores, ld, row_len, tok_pos, K, idx, err);
  return counted(cudaGetLastError());
}

}  // namespace dsa
