// Top-K selection ([P3] "Inference Acceleration for a New Domestic LLM
// Architecture...", section 3 `topk_select`; [P2] "Hybrid Attention LLM
// Inference Acceleration...", section 2 item 2).
//
// Per row: the min(K, n) positions with the largest scores, equal scores ->
// lower position, emitted in ascending position order, padded with -1.  No
// sort of the row is ever materialised.
//
// Scores map to order-preserving 32-bit keys (-0.0 folded to +0.0 first).
//   1. histogram of the top 11 key bits (2048 bins; lanes of a warp that hit
//      the same bin add once) -> the bin b* that holds the K-th largest key,
//      and k_rem = how many of b*'s members are still needed;
//   2. one ordered pass: positions in bins above b* are "sure" (fewer than K),
//      positions in b* are candidates; both lists stay in position order;
//   3. radix select on the low 21 bits (3 x 7 bits) among the candidates
//      gives the exact key tau of the K-th largest and r = the number of
//      tau-valued candidates taken (the lowest positions);
//   4. the selected candidates are merged with the sure list by position.
// Rows much longer than the number of rows get several CTAs per row
// (histogram -> filter -> select kernels); otherwise one CTA does a row.
// A degenerate row whose threshold bin holds more candidates than shared
// memory falls back to four 8-bit radix passes over the whole row.
#include "dsa_internal.cuh"

namespace dsa {

namespace {

constexpr int kHistBins = kTopkHistBins;  // top 11 key bits
constexpr int kLowBits = kTopkLowBits;
constexpr int kRowThreads = 1024;
constexpr int kCandCap = 12288;      // candidates kept in shared memory by the one-CTA path
constexpr int kChunkThreads = 512;

// Exclusive block-wide prefix sum of v (blockDim.x a multiple of 32, <= 1024);
// *total receives the sum.  Uses the 33-word scratch `buf`.
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
  if (warp == 0) {
    const uint32_t w = lane < nw ? buf[lane] : 0u;
    uint32_t wi = w;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, wi, o);
      if (lane >= o) wi += u;
    }
    buf[lane] = wi - w;
    if (lane == 31) buf[32] = wi;
  }
  __syncthreads();
  const uint32_t r = buf[warp] + incl - v;
  *total = buf[32];
  __syncthreads();
  return r;
}

// In a histogram of `bins` bins (bins a multiple of 32), find d such that the
// keys above d number `above` < need <= above + hist[d].  Warp 0 computes;
// the result is broadcast through shared memory.
__device__ __forceinline__ void find_bin(const uint32_t* hist, int bins, uint32_t need, uint32_t* out_bin,
                                         uint32_t* out_above) {
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    const int per = bins / 32;
    const int top = bins - 1 - lane * per;  // lane covers top .. top-per+1
    uint32_t sum = 0;
    for (int j = 0; j < per; ++j) sum += hist[top - j];
    uint32_t incl = sum;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t u = __shfl_up_sync(0xffffffffu, incl, o);
      if (lane >= o) incl += u;
    }
    const uint32_t excl = incl - sum;
    if (excl < need && need <= incl) {
      uint32_t above = excl;
      for (int j = 0; j < per; ++j) {
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
  __syncthreads();
}

// Exact key tau of the `need`-th largest candidate key (all candidates share
// the top 11 bits `top`) and r = tau-valued candidates to take.  Keys come
// from get_key(i), i < m.
template <class GetKey>
__device__ __forceinline__ void select_among(int m, uint32_t need, uint32_t top, GetKey get_key, uint32_t* hist128,
                                             uint32_t* s_bin, uint32_t* s_above, uint32_t* tau_out,
                                             uint32_t* r_out) {
  uint32_t prefix = top << kLowBits, mask = 0xFFFFFFFFu << kLowBits;
  for (int pass = 0; pass < 3; ++pass) {
    const int shift = 14 - 7 * pass;
    for (int i = threadIdx.x; i < 128; i += blockDim.x) hist128[i] = 0;
    __syncthreads();
    for (int base = 0; base < m; base += blockDim.x) {
      const int i = base + threadIdx.x;
      uint32_t key = 0;
      bool act = false;
      if (i < m) {
        key = get_key(i);
        act = (key & mask) == prefix;
      }
      hist_add(hist128, (key >> shift) & 127u, act);
    }
    __syncthreads();
    find_bin(hist128, 128, need, s_bin, s_above);
    prefix |= *s_bin << shift;
    mask |= 127u << shift;
    need -= *s_above;
    __syncthreads();
  }
  *tau_out = prefix;
  *r_out = need;
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

// Merge two ascending, disjoint position lists into out[0 .. na+nb).
__device__ __forceinline__ void merge_lists(const int32_t* A, int na, const int32_t* B, int nb, int32_t* out) {
  for (int i = threadIdx.x; i < na; i += blockDim.x) {
    const int32_t v = A[i];
    int lo = 0, hi = nb;  // number of B elements below v
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (B[mid] < v) lo = mid + 1; else hi = mid;
    }
    out[i + lo] = v;
  }
  for (int j = threadIdx.x; j < nb; j += blockDim.x) {
    const int32_t v = B[j];
    int lo = 0, hi = na;
    while (lo < hi) {
      const int mid = (lo + hi) >> 1;
      if (A[mid] < v) lo = mid + 1; else hi = mid;
    }
    out[j + lo] = v;
  }
}

__device__ __forceinline__ int row_length(const int32_t* row_len, const int32_t* tok_pos, int t, int64_t ld,
                                          uint32_t* err) {
  const int64_t n64 = row_len ? (int64_t)row_len[t] : (int64_t)tok_pos[t] + 1;
  if (row_len && (n64 < 0 || n64 > ld)) raise_error(err, kErrBadIndex);
  return (int)(n64 < 0 ? 0 : (n64 > ld ? ld : n64));
}

// Selected candidates of a row in position order: keys above tau, and the
// first r keys equal to tau.  pos_of(i) / key_of(i) give candidate i.
template <class PosOf, class KeyOf>
__device__ __forceinline__ void emit_selected(int m, uint32_t tau, uint32_t r, uint32_t need, PosOf pos_of,
                                              KeyOf key_of, int32_t* sel, uint32_t* buf) {
  uint32_t run_gt = 0, run_eq = 0;
  for (int base = 0; base < m; base += blockDim.x * 4) {
    const int i0 = base + threadIdx.x * 4;
    uint32_t gt = 0, eq = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (i0 + j < m) {
        const uint32_t key = key_of(i0 + j);
        gt |= (uint32_t)(key > tau) << j;
        eq |= (uint32_t)(key == tau) << j;
      }
    const TwoLists L = scan_two(gt, eq, run_gt, run_eq, buf);
    uint32_t eq_before = L.pb;
    uint32_t p = L.pa + min(eq_before, r);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (gt >> j & 1u) {
        if (p < need) sel[p] = pos_of(i0 + j);
        ++p;
      } else if (eq >> j & 1u) {
        if (eq_before < r) {
          if (p < need) sel[p] = pos_of(i0 + j);
          ++p;
        }
        ++eq_before;
      }
    }
    run_gt += L.ta;
    run_eq += L.tb;
  }
  __syncthreads();
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
    find_bin(hist, 256, need, s_bin, s_above);
    prefix |= *s_bin << shift;
    mask |= 0xFFu << shift;
    need -= *s_above;
    __syncthreads();
  }
  // every key > tau and the first `need` keys == tau, straight into out
  emit_selected(
      n, prefix, need, (uint32_t)K, [&](int i) { return (int32_t)i; }, [&](int i) { return order_key(row[i]); },
      out, buf);
}

// ---------------------------------------------------------------- one CTA per row
struct RowSmem {
  uint32_t hist[kHistBins];
  uint32_t hist128[128];
  uint32_t buf[33];
  uint32_t bin, above;
  int32_t sure[kMaxK];
  int32_t sel[kMaxK];
  int32_t cand_idx[kCandCap];
  uint32_t cand_key[kCandCap];
};

__global__ void __launch_bounds__(kRowThreads)
k_topk_row(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
           const int32_t* __restrict__ tok_pos, int K, int32_t* __restrict__ idx, uint32_t* err) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  RowSmem& sm = *reinterpret_cast<RowSmem*>(smem_raw);
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
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sm.hist[i] = 0;
  __syncthreads();
  for (int base = 0; base < n; base += blockDim.x) {
    const int s = base + threadIdx.x;
    const bool act = s < n;
    const uint32_t key = act ? order_key(row[s]) : 0u;
    hist_add(sm.hist, key >> kLowBits, act);
  }
  __syncthreads();
  find_bin(sm.hist, kHistBins, (uint32_t)K, &sm.bin, &sm.above);
  const uint32_t bstar = sm.bin, above = sm.above;
  const uint32_t m = sm.hist[bstar];
  __syncthreads();
  if (m > (uint32_t)kCandCap) {  // degenerate distribution: exact radix over the whole row
    topk_row_full_radix(row, n, K, out, sm.hist, sm.buf, &sm.bin, &sm.above);
    return;
  }
  // sure list (bins above b*) and candidate list (bin b*), in position order
  uint32_t run_s = 0, run_c = 0;
  for (int base = 0; base < n; base += blockDim.x * 4) {
    const int s0 = base + threadIdx.x * 4;
    uint32_t sa = 0, cb = 0, keys[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      keys[j] = 0;
      if (s0 + j < n) {
        keys[j] = order_key(row[s0 + j]);
        const uint32_t bin = keys[j] >> kLowBits;
        sa |= (uint32_t)(bin > bstar) << j;
        cb |= (uint32_t)(bin == bstar) << j;
      }
    }
    const TwoLists L = scan_two(sa, cb, run_s, run_c, sm.buf);
    uint32_t ps = L.pa, pc = L.pb;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (sa >> j & 1u) {
        if (ps < (uint32_t)kMaxK) sm.sure[ps] = s0 + j;
        ++ps;
      } else if (cb >> j & 1u) {
        if (pc < (uint32_t)kCandCap) {
          sm.cand_idx[pc] = s0 + j;
          sm.cand_key[pc] = keys[j];
        }
        ++pc;
      }
    }
    run_s += L.ta;
    run_c += L.tb;
  }
  __syncthreads();
  const uint32_t need = (uint32_t)K - above;
  uint32_t tau, r;
  select_among(
      (int)m, need, bstar, [&](int i) { return sm.cand_key[i]; }, sm.hist128, &sm.bin, &sm.above, &tau, &r);
  emit_selected(
      (int)m, tau, r, need, [&](int i) { return sm.cand_idx[i]; }, [&](int i) { return sm.cand_key[i]; }, sm.sel,
      sm.buf);
  merge_lists(sm.sure, (int)above, sm.sel, (int)need, out);
}

// ---------------------------------------------------------------- several CTAs per row
// Scratch per call: hist [T][2048] (zeroed before k_topk_hist), counts
// [T][C] {sure, cand}, sure lists [T][C][K], candidate lists [T][C][chunk].

__global__ void __launch_bounds__(kChunkThreads)
k_topk_hist(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
            const int32_t* __restrict__ tok_pos, int K, int chunk, uint32_t* __restrict__ ghist, uint32_t* err) {
  __shared__ uint32_t hist[kHistBins];
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y, c = blockIdx.x;
  const int n = row_length(row_len, tok_pos, t, ld, err);
  const int b0 = c * chunk, b1 = min(n, b0 + chunk);
  if (n <= K || b0 >= b1) return;
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) hist[i] = 0;
  __syncthreads();
  const float* __restrict__ row = scores + (int64_t)t * ld;
  for (int base = b0; base < b1; base += blockDim.x) {
    const int s = base + threadIdx.x;
    const bool act = s < b1;
    const uint32_t key = act ? order_key(row[s]) : 0u;
    hist_add(hist, key >> kLowBits, act);
  }
  __syncthreads();
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x)
    if (hist[i]) atomicAdd(&ghist[(int64_t)t * kHistBins + i], hist[i]);
}

constexpr int kMaxChunks = 64;
constexpr int kSelCap = 4096;  // candidates staged in shared memory by the select step

struct SelSmem {
  uint32_t hist[kHistBins];
  uint32_t hist128[128];
  uint32_t buf[33];
  uint32_t bin, above;
  int sure_off[kMaxChunks + 1], cand_off[kMaxChunks + 1];
  int32_t sure[kMaxK];
  int32_t sel[kMaxK];
  int32_t cpos[kSelCap];
  uint32_t ckey[kSelCap];
  int last;
};

// Index of the last offset <= i in off[0..C-1] (off ascending).
__device__ __forceinline__ int chunk_of(const int* off, int C, int i) {
  int lo = 0, hi = C - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= i) lo = mid; else hi = mid - 1;
  }
  return lo;
}

// Exact selection for row t once every chunk of it has been filtered.  The
// lists were written by other CTAs of this grid: read through L2 (__ldcg).
// Every global read is issued in parallel (no chains over chunks).
__device__ void select_row(int t, const float* __restrict__ row, int K, int chunk, int C,
                           const uint32_t* __restrict__ ghist, const int2* __restrict__ counts,
                           const int32_t* __restrict__ sure, const int32_t* __restrict__ cand,
                           int32_t* __restrict__ out, SelSmem& sm) {
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sm.hist[i] = __ldcg(ghist + (int64_t)t * kHistBins + i);
  if (threadIdx.x < 64) {  // chunk counts -> offsets: two lanes' worth per thread of warps 0-1, scanned by warp 0
    const int2 v = threadIdx.x < C ? __ldcg(counts + (int64_t)t * C + threadIdx.x) : make_int2(0, 0);
    sm.sure_off[threadIdx.x + 1] = v.x;
    sm.cand_off[threadIdx.x + 1] = v.y;
  }
  __syncthreads();
  if (threadIdx.x < 32) {
    const int lane = threadIdx.x;
    int a0 = sm.sure_off[2 * lane + 1], a1 = sm.sure_off[2 * lane + 2];
    int c0 = sm.cand_off[2 * lane + 1], c1 = sm.cand_off[2 * lane + 2];
    int sa = a0 + a1, sc = c0 + c1;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int ua = __shfl_up_sync(0xffffffffu, sa, o), uc = __shfl_up_sync(0xffffffffu, sc, o);
      if (lane >= o) { sa += ua; sc += uc; }
    }
    // sa / sc are inclusive sums through element 2*lane+1
    sm.sure_off[2 * lane + 2] = sa;
    sm.sure_off[2 * lane + 1] = sa - a1;
    sm.cand_off[2 * lane + 2] = sc;
    sm.cand_off[2 * lane + 1] = sc - c1;
    if (lane == 0) {
      sm.sure_off[0] = 0;
      sm.cand_off[0] = 0;
    }
  }
  __syncthreads();
  find_bin(sm.hist, kHistBins, (uint32_t)K, &sm.bin, &sm.above);
  const uint32_t bstar = sm.bin, above = sm.above;
  const uint32_t need = (uint32_t)K - above;
  const int m = sm.cand_off[C];
  const int A = min(sm.sure_off[C], kMaxK);
  // the sure list, concatenated in chunk order (already ascending)
  for (int i = threadIdx.x; i < A; i += blockDim.x) {
    const int c = chunk_of(sm.sure_off, C, i);
    sm.sure[i] = __ldcg(sure + ((int64_t)t * C + c) * K + (i - sm.sure_off[c]));
  }
  // candidate i of the row-wide list lives in chunk c at offset i - cand_off[c]
  auto cand_pos = [&](int i) -> int32_t {
    const int c = chunk_of(sm.cand_off, C, i);
    return __ldcg(cand + ((int64_t)t * C + c) * chunk + (i - sm.cand_off[c]));
  };
  uint32_t tau, r;
  if (m <= kSelCap) {
    for (int i = threadIdx.x; i < m; i += blockDim.x) {
      const int32_t pos = cand_pos(i);
      sm.cpos[i] = pos;
      sm.ckey[i] = order_key(row[pos]);
    }
    __syncthreads();
    select_among(
        m, need, bstar, [&](int i) { return sm.ckey[i]; }, sm.hist128, &sm.bin, &sm.above, &tau, &r);
    emit_selected(
        m, tau, r, need, [&](int i) { return sm.cpos[i]; }, [&](int i) { return sm.ckey[i]; }, sm.sel, sm.buf);
  } else {
    __syncthreads();
    select_among(
        m, need, bstar, [&](int i) { return order_key(row[cand_pos(i)]); }, sm.hist128, &sm.bin, &sm.above, &tau,
        &r);
    emit_selected(
        m, tau, r, need, cand_pos, [&](int i) { return order_key(row[cand_pos(i)]); }, sm.sel, sm.buf);
  }
  merge_lists(sm.sure, (int)above, sm.sel, (int)need, out);
}

// Filters chunk c of row t into its sure and candidate lists; the CTA that
// finishes a row's last chunk then selects that row.
__global__ void __launch_bounds__(kChunkThreads)
k_topk_filter_select(const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ row_len,
                     const int32_t* __restrict__ tok_pos, int K, int chunk, int C, const uint32_t* __restrict__ ghist,
                     int2* __restrict__ counts, int32_t* __restrict__ sure, int32_t* __restrict__ cand,
                     int* __restrict__ row_done, int32_t* __restrict__ idx) {
  extern __shared__ __align__(16) unsigned char smem_raw[];
  SelSmem& sm = *reinterpret_cast<SelSmem*>(smem_raw);
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y, c = blockIdx.x;
  const int n = row_length(row_len, tok_pos, t, ld, nullptr);
  int32_t* __restrict__ out = idx + (int64_t)t * K;
  if (n <= K) {  // every candidate is selected
    if (c == 0)
      for (int i = threadIdx.x; i < K; i += blockDim.x) out[i] = i < n ? i : -1;
    return;
  }
  const int b0 = c * chunk, b1 = min(n, b0 + chunk);
  for (int i = threadIdx.x; i < kHistBins; i += blockDim.x) sm.hist[i] = __ldcg(ghist + (int64_t)t * kHistBins + i);
  __syncthreads();
  find_bin(sm.hist, kHistBins, (uint32_t)K, &sm.bin, &sm.above);
  const uint32_t bstar = sm.bin;
  const float* __restrict__ row = scores + (int64_t)t * ld;
  int32_t* my_sure = sure + ((int64_t)t * C + c) * K;
  int32_t* my_cand = cand + ((int64_t)t * C + c) * chunk;
  uint32_t run_s = 0, run_c = 0;
  for (int base = b0; base < b1; base += blockDim.x * 4) {
    const int s0 = base + threadIdx.x * 4;
    uint32_t sa = 0, cb = 0;
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < b1) {
        const uint32_t bin = order_key(row[s0 + j]) >> kLowBits;
        sa |= (uint32_t)(bin > bstar) << j;
        cb |= (uint32_t)(bin == bstar) << j;
      }
    const TwoLists L = scan_two(sa, cb, run_s, run_c, sm.buf);
    uint32_t ps = L.pa, pc = L.pb;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      if (sa >> j & 1u) {
        if (ps < (uint32_t)K) my_sure[ps] = s0 + j;
        ++ps;
      } else if (cb >> j & 1u) {
        my_cand[pc++] = s0 + j;
      }
    }
    run_s += L.ta;
    run_c += L.tb;
  }
  __syncthreads();  // every list write of this CTA precedes the count
  if (threadIdx.x == 0) {
    counts[(int64_t)t * C + c] = make_int2((int)run_s, (int)run_c);
    __threadfence();
    sm.last = atomicAdd(&row_done[t], 1) == C - 1;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();  // the other chunks' lists are visible from here on
  select_row(t, row, K, chunk, C, ghist, counts, sure, cand, out, sm);
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

}  // namespace

// Scratch layout (several CTAs per row): a region zeroed on every call --
// row_done [T] (padded to 16 words) then the first-digit histogram [T][2048]
// -- followed by counts [T][C], sure lists [T][C][K] and candidates [T][C][chunk].
int64_t topk_zero_words(int T) { return (int64_t)(T + 15) / 16 * 16 + (int64_t)T * kHistBins; }

size_t topk_scratch_bytes(int T, int64_t ld, int K) {
  int C, chunk;
  topk_chunks(T, ld, &C, &chunk);
  if (C == 1) return 0;
  return (size_t)topk_zero_words(T) * 4 + (size_t)T * C * sizeof(int2) + (size_t)T * C * K * 4 +
         (size_t)T * C * chunk * 4;
}

uint32_t* topk_hist_in_scratch(void* scratch, int T) {
  return reinterpret_cast<uint32_t*>(scratch) + (T + 15) / 16 * 16;
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
    e = launch_pdl(k_topk_row, dim3(T), dim3(kRowThreads), sizeof(RowSmem), st, scores, ld, row_len, tok_pos, K, idx,
                   err);
    if (e != cudaSuccess) return e;
    return counted(cudaGetLastError());
  }
  int* row_done = reinterpret_cast<int*>(scratch);
  uint32_t* ghist = topk_hist_in_scratch(scratch, T);
  char* p = reinterpret_cast<char*>(scratch) + topk_zero_words(T) * 4;
  int2* counts = reinterpret_cast<int2*>(p);
  p += (size_t)T * C * sizeof(int2);
  int32_t* sure = reinterpret_cast<int32_t*>(p);
  p += (size_t)T * C * K * 4;
  int32_t* cand = reinterpret_cast<int32_t*>(p);
  cudaError_t e = cudaSuccess;
  const dim3 grid(C, T);
  if (!hist_ready) {  // otherwise the caller has zeroed the region and filled the histogram
    if ((e = cudaMemsetAsync(scratch, 0, (size_t)topk_zero_words(T) * 4, st)) != cudaSuccess) return e;
    e = launch_pdl(k_topk_hist, grid, dim3(kChunkThreads), 0, st, scores, ld, row_len, tok_pos, K, chunk, ghist, err);
    if (e != cudaSuccess || (e = counted(cudaGetLastError())) != cudaSuccess) return e;
  }
  static thread_local int dev_fs = -1;
  if ((e = set_smem_once(k_topk_filter_select, (int)sizeof(SelSmem), &dev_fs)) != cudaSuccess) return e;
  e = launch_pdl(k_topk_filter_select, grid, dim3(kChunkThreads), sizeof(SelSmem), st, scores, ld, row_len, tok_pos, K,
                 chunk, C, (const uint32_t*)ghist, counts, sure, cand, row_done, idx);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace dsa
