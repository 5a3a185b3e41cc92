// Radix-select building blocks shared by the Top-K kernels (k_topk.cu) and
// the indexer's fused selection tail (k_indexer.cu).  The order-preserving
// 32-bit key of a score is resolved as three digits: bits 31..21 (2048
// bins), 20..10 (2048 bins) and 9..0 (1024 bins).
#pragma once
#include "dsa_internal.cuh"

namespace dsa {
namespace topk {

constexpr int kD1Bins = kTopkHistBins;  // digit 1: key bits 31..21
constexpr int kD2Bins = 2048;           // digit 2: key bits 20..10
constexpr int kD3Bins = 1024;           // digit 3: key bits 9..0

__device__ __forceinline__ uint32_t digit1(uint32_t key) { return key >> kTopkLowBits; }
__device__ __forceinline__ uint32_t digit2(uint32_t key) { return (key >> 10) & (kD2Bins - 1); }
__device__ __forceinline__ uint32_t digit3(uint32_t key) { return key & (kD3Bins - 1); }

// Exclusive block-wide prefix sum of v (blockDim.x a multiple of 32, <= 1024);
// *total receives the sum.  Each warp scans its own values; the warp totals
// go through `buf` (32 words) and every warp reduces them itself -- two
// barriers and no second serial scan.
__device__ __forceinline__ uint32_t block_scan(uint32_t v, uint32_t* buf, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  uint32_t incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  if (lane == 31) buf[warp] = incl;
  __syncthreads();
  const uint32_t x = lane < nw ? buf[lane] : 0u;
  uint32_t below = lane < warp ? x : 0u, all = x;  // totals of the earlier warps / of every warp
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    below += __shfl_xor_sync(0xffffffffu, below, o);
    all += __shfl_xor_sync(0xffffffffu, all, o);
  }
  *total = all;
  __syncthreads();  // buf is free for the next scan
  return below + incl - v;
}

// In a histogram of `bins` bins (a power of two, 256 .. 2048), find d such
// that the keys above d number `above` < need <= above + hist[d].  Warp 0
// alone: lane l sums the bins [l*per, l*per + per) (rotated reads, no bank
// conflicts), a suffix scan over the lanes finds the lane holding the
// crossing, and a second pass splits that lane's bins over the warp.  If no
// bin qualifies (need 0 or above the total) the result is bin 0 with nothing
// above it.  Ends with a barrier.
template <int BINS>
__device__ __forceinline__ void find_bin(const uint32_t* hist, uint32_t need, uint32_t* out_bin, uint32_t* out_above) {
  static_assert(BINS >= 256 && BINS <= 2048 && (BINS & (BINS - 1)) == 0, "bins");
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    constexpr int per = BINS >> 5;
    uint32_t v[per];  // every load issued before the sums
#pragma unroll
    for (int j = 0; j < per; ++j) v[j] = hist[lane * per + ((j + lane) & (per - 1))];
    uint32_t sum = 0;
#pragma unroll
    for (int j = 0; j < per; ++j) sum += v[j];
    uint32_t incl = sum;  // keys in this lane's bins and every higher lane's
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_down_sync(0xffffffffu, incl, o);
      if (lane + o < 32) incl += u;
    }
    const uint32_t who = __ballot_sync(0xffffffffu, incl - sum < need && need <= incl);
    if (who == 0) {
      if (lane == 0) {
        *out_bin = 0u;
        *out_above = 0u;
      }
    } else {
      const int L = __ffs(who) - 1;
      const uint32_t above_l = __shfl_sync(0xffffffffu, incl - sum, L);
      constexpr int q = per >= 32 ? per >> 5 : 1;  // bins per lane in the second pass
      const int top = L * per + per - 1 - lane * q;  // this lane's bins: top, top-1, ..., top-q+1
      const bool mine = lane * q < per;
      uint32_t s2 = 0;
      if (mine) {
#pragma unroll
        for (int j = 0; j < q; ++j) s2 += hist[top - j];
      }
      uint32_t inc2 = s2;  // from the top of L's range down to this lane's bins
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t u = __shfl_up_sync(0xffffffffu, inc2, o);
        if (lane >= o) inc2 += u;
      }
      const uint32_t ex = above_l + inc2 - s2;
      if (mine && s2 != 0 && ex < need && need <= ex + s2) {
        uint32_t above = ex;
#pragma unroll
        for (int j = 0; j < q; ++j) {
          const uint32_t c = hist[top - j];
          if (above + c >= need) {
            *out_bin = (uint32_t)(top - j);
            *out_above = above;
            break;
          }
          above += c;
        }
      }
    }
  }
  __syncthreads();
}

// Ordered compaction of (at most) 4 consecutive elements per thread into two
// lists: bit j of `a` / `b` says element j goes to list A / B.  Returns the
// thread's first positions in each list (running offsets added) and totals.
struct TwoLists {
  uint32_t pa, pb, ta, tb;
};
__device__ __forceinline__ TwoLists scan_two(uint32_t a, uint32_t b, uint32_t run_a, uint32_t run_b, uint32_t* buf) {
  uint32_t total;
  const uint32_t packed = ((uint32_t)__popc(a) << 16) | (uint32_t)__popc(b);
  const uint32_t excl = block_scan(packed, buf, &total);
  return {run_a + (excl >> 16), run_b + (excl & 0xFFFFu), total >> 16, total & 0xFFFFu};
}

// Emits, in the order of the list, the position of every element whose key is
// > tau and of the first r elements whose key == tau (at most K positions are
// written).  get(i) -> {position, key} for i < L.
template <class Get>
__device__ __forceinline__ void emit_selected(int L, uint32_t tau, uint32_t r, int K, Get get, int32_t* out,
                                              uint32_t* buf) {
  uint32_t run_gt = 0, run_eq = 0;
  for (int base = 0; base < L; base += blockDim.x * 4) {
    const int i0 = base + threadIdx.x * 4;
    uint32_t gt = 0, eq = 0;
    int2 e[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) e[j] = i0 + j < L ? get(i0 + j) : make_int2(0, 0);
    int32_t pos[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      pos[j] = e[j].x;
      if (i0 + j < L) {
        gt |= (uint32_t)((uint32_t)e[j].y > tau) << j;
        eq |= (uint32_t)((uint32_t)e[j].y == tau) << j;
      }
    }
    const TwoLists S = scan_two(gt, eq, run_gt, run_eq, buf);
    uint32_t eq_before = S.pb;
    uint32_t p = S.pa + min(eq_before, r);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (gt >> j & 1u) {
        if (p < (uint32_t)K) out[p] = pos[j];
        ++p;
      } else if (eq >> j & 1u) {
        if (eq_before < r) {
          if (p < (uint32_t)K) out[p] = pos[j];
          ++p;
        }
        ++eq_before;
      }
    }
    run_gt += S.ta;
    run_eq += S.tb;
  }
}

}  // namespace topk
}  // namespace dsa
