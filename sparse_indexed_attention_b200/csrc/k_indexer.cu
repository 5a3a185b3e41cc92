// Lightweight-indexer scores on the 5th-generation tensor cores
// ([P2] "Hybrid Attention LLM Inference Acceleration...", section 2 item 2 and
// section 4(1): scoring + head weighting read the paged K cache directly;
// [P4] "Optimizing Inference for Hybrid-Architecture Large Language
// Models...", section 3.1):
//
//   score[t,s] = kI_scale[s] * sum_h w'[t,h] * ReLU(q^[t,h,:] . k^[s,:])
//
// As a GEMM per (token group, key tile): D[s, (t,h)] = sum_d K[s,d] Q[(t,h),d]
// with M = 128 keys (two 64-row pages), N = 64 heads x TG tokens, K = 128.
//  * warp 0, one lane: TMA producer.  Each key tile is two TMA loads of one
//    8 KB page each, straight from the paged pool (the page table is read
//    here), plus a 256-byte bulk copy of each page's row scales.  The group's
//    quantized query rows and head weights are loaded once per group.
//  * warp 1, one lane: issues tcgen05.mma (kind::f8f6f4 E4M3, or kind::f16
//    bf16) into a ring of TMEM accumulators; tcgen05.commit frees the stage
//    and publishes the accumulator.
//  * MXFP8 cache ([P2] section 5 table, "Indexer Q/K": one shared scale per
//    group of 32; [P4] section 4.2): keys and the quantized query carry one
//    E8M0 scale per 32 of the 128 dims, applied by the tensor core itself
//    (kind::mxf8f6f4.block_scale, one MMA per 32-wide K block).  The
//    producer warp's 32 lanes copy a tile's key scales (4-byte cp.async) into
//    shared memory in the scale-factor layout -- key r in row r % 32, 32-bit
//    column r / 32, byte = K block -- and a group's query scales likewise;
//    the MMA lane moves them into TMEM with tcgen05.cp (32 rows x 128 bits,
//    written to every lane quarter) ahead of the tile's MMAs.  The epilogue
//    is that of the E4M3 cache without the key scale.
//  * warp 2: allocates and frees TMEM.
//  * warps 4-11: epilogue, two warpgroups taking alternate tiles.  Thread r
//    of a warpgroup owns TMEM lane r = key row r, so the ReLU, the head
//    weighting and the reduction over heads stay inside one thread; no
//    [T, H_I, N] value ever leaves the SM.
// The CTA grid is persistent (one CTA per SM) over the work items of k_plan.
//
// Decode (one token per group) can also select the Top-K inside the same
// kernel, the fused scoring-weighting-selection operator of [P2] section 4(1)
// and [P4] section 3.1: the epilogue keeps every score of the CTA's items in
// shared memory as its order-preserving key (no score ever reaches global
// memory), and once a CTA has scored its items it resolves, together with
// the other CTAs holding parts of the same rows, the K-th largest key of
// each row digit by digit (11, 11 and 10 bits) through per-row histograms in
// global memory, then writes its own selections, ascending, at offsets
// derived from per-item counts.  Rows meet through arrival counters with
// bounded waits; the persistent grid (one CTA per SM) is all resident.
#include <cudaTypedefs.h>

#include "sm100.cuh"
#include "topk_select.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kEpiWarps = 8;                 // two epilogue warpgroups (warps 4-11)
constexpr int kRingSlots = 8;                // producer's look-ahead ring (items)
constexpr int kRecAhead = 6;                 // item records are fetched this many items ahead
constexpr int kPgAhead = 3;                  // page ids this many items ahead
constexpr int kIdxThreads = (4 + kEpiWarps) * 32;

constexpr int kTailRuns = 32;                // rows a CTA can hold parts of (fused selection)
constexpr int kTailItemsMax = 32;            // items a CTA can keep the scores of (fused selection)

// Fast path of the fused selection: a row's candidates (keys whose first
// digit reaches the row's threshold bin, typically a little over K) go to one
// list per row that the CTA holding the row's last item resolves alone; it
// emits the selected positions in order through two bitmaps over the row.
constexpr int kCandCap = 6144;               // candidates per row
constexpr int kBitmapWords = 4608;           // rows of up to 147,456 positions
constexpr int kFastScratch = kCandCap * 8 + 2 * kBitmapWords * 4;  // in the score-key area

// Shared-memory scratch of the fused selection tail.
struct TailSmem {
  uint32_t hist[kTopkHistBins];
  uint32_t buf[33];
  uint32_t bin, above;
  int nruns, bad;
  uint32_t red[8];
  int4 item_info[kTailItemsMax];  // per item of the CTA: {token, position, tile begin, tile end}
  int4 runs[kTailRuns];          // {token, first item, end item, position}
  uint32_t prefix[kTailRuns];    // resolved high digits of the row's K-th key
  uint32_t need[kTailRuns];      // selections still to find below the resolved digits
  uint32_t ncand[kTailRuns];     // candidates of the row (first digit at or above its threshold bin)
  int fast[kTailRuns];           // the row takes the candidate-list path
};

template <bool kBf16, int TG, bool kFused = false, bool kMx = false>
struct IdxCfg {
  static_assert(!kFused || TG == 1, "the fused selection serves one token per group");
  static_assert(!kMx || (!kBf16 && TG <= 2), "MXFP8: E4M3 codes, at most two tokens per group");
  static constexpr int N = 64 * TG;                        // MMA N: heads x tokens of a group
  static constexpr int A_BYTES = kBf16 ? 32768 : 16384;    // 128 keys x d_I
  static constexpr int B_BYTES = kBf16 ? N * 256 : N * 128;
  static constexpr int KSTEPS = kBf16 ? 8 : 4;             // 32-byte K steps per tile
  static constexpr int NS = kBf16 ? 3 : (TG == 1 ? (kFused ? 6 : 8) : 6);
  // Accumulator ring.  NACC is even: the two epilogue warpgroups take
  // alternate tiles, so each accumulator (and its barriers) belongs to one
  // warpgroup and is waited on one phase at a time.  MXFP8 also keeps scale
  // columns in TMEM: 4 per stage (128 keys), 4 per group slot and 128 query rows.
  static constexpr int NACC = kMx ? (N == 64 ? 4 : 2) : ((512 / N) < 4 ? (512 / N) : 4);
  static constexpr int SFB_COPIES = kMx ? (N + 127) / 128 : 0;   // 32x128b copies per group
  static constexpr int SFB_BYTES = SFB_COPIES * 512;
  static constexpr int SFA0 = NACC * N;                    // TMEM column of stage 0's key scales
  static constexpr int SFB0 = SFA0 + 4 * NS;               // TMEM column of slot 0's query scales
  static constexpr int SFB_COLS = 4 * SFB_COPIES;
  static constexpr int TMEM_COLS = kMx ? 512 : ((NACC * N) <= 256 ? 256 : 512);
  // shared-memory layout (offsets from a 1024-aligned base)
  static constexpr int OFF_A = 0;
  static constexpr int OFF_B = OFF_A + NS * A_BYTES;
  static constexpr int OFF_SC = OFF_B + 2 * B_BYTES;       // NS x 128 fp32 row scales
  static constexpr int OFF_W = OFF_SC + NS * 512;          // 2 x TG x 64 fp32 head weights
  // (MXFP8: the OFF_SC area holds each stage's key scales in the scale-factor layout, 512 B)
  static constexpr int OFF_SFB = OFF_W + 2 * TG * 256;    // MXFP8: 2 x the group's query scales
  static constexpr int OFF_HIST = OFF_SFB + 2 * SFB_BYTES;  // TG == 1: per-epilogue-warp Top-K histograms
  static constexpr int OFF_RING = OFF_HIST + ((TG == 1 && !kFused) ? kEpiWarps * kTopkHistBins * 4 : 0);
  static constexpr int OFF_BAR = OFF_RING + kRingSlots * (32 + 128);  // producer's item records + page ids
  static constexpr int NBARS = 2 * NS + 4 + 2 * NACC + 1;
  static constexpr int OFF_MISC = OFF_BAR + NBARS * 8;
  static constexpr int OFF_TAIL = (OFF_MISC + 16 + 15) / 16 * 16;     // fused: selection scratch
  static constexpr int OFF_KEYS = OFF_TAIL + (kFused ? (int)((sizeof(TailSmem) + 15) / 16 * 16) : 0);
  // fused: score keys of up to CAP_ITEMS items (1024 keys each) in shared memory
  static constexpr int CAP_RAW = kFused ? (227 * 1024 - 1024 - OFF_KEYS) / 4096 : 0;
  static constexpr int CAP_ITEMS = CAP_RAW < kTailItemsMax ? CAP_RAW : kTailItemsMax;
  static constexpr int BYTES = OFF_KEYS + CAP_ITEMS * 4096;
  static constexpr int SMEM = BYTES + 1024;                // slack for 1024-byte alignment
  static constexpr uint32_t IDESC = make_idesc(kBf16, 128, N);
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(NACC * N <= TMEM_COLS && NACC % 2 == 0, "TMEM accumulators (an even number)");
  static_assert(!kMx || SFB0 + 2 * SFB_COLS <= TMEM_COLS, "TMEM scale columns");
  static_assert(OFF_SFB % 512 == 0, "scale-factor sources need 16-byte alignment");
  static_assert(!kFused || CAP_ITEMS >= 8, "fused selection capacity");
  static_assert(!kFused || CAP_ITEMS * 4096 >= kFastScratch, "fused selection fast-path scratch");
};

struct IdxArgs {
  SeqsDev s;
  PlanBufs plan;
  const float* w_operand;  // [T, 64] head weights (scaled by 2^e for FP8)
  const float* kI_scale;   // [R] (FP8) or null
  const uint8_t* kI_sf;    // MXFP8: key group scales [R, 4] (E8M0)
  const uint8_t* q_sf;     // MXFP8: query group scales [T * 64, 4] (E8M0)
  float* scores;
  int64_t ld;
  uint32_t* hist;          // TG == 1 only, may be null: Top-K first-digit histogram [T][2048]
  uint32_t* err;
  uint64_t wait_ns;        // limit of each wait for another role's progress
  // fused selection (zeroed by the call's prep kernel): per token
  // [digit-1 hist 2048][digit-2 hist 2048][digit-3 hist 1024][arrivals 4][pad 4],
  // then per item {keys > tau, keys == tau} of its CTA's run
  uint32_t* tail;
  int2* tail_items;
  int2* cand;              // [T][kCandCap] (position, key) candidates, not zeroed
  int32_t* idx;            // [T, K] selected positions
  int K;
};

constexpr int kTailWords = kFusedTailWordsPerToken;  // per token
static_assert(kTailWords == 2 * kTopkHistBins + topk::kD3Bins + 8, "fused tail layout");
constexpr int kTailArrive = 2 * kTopkHistBins + topk::kD3Bins;  // 4 arrival counters
constexpr int kTailCandCount = kTailArrive + 4;                  // candidates published so far

// Waits (bounded) until the arrival counter at p has reached target.
__device__ __forceinline__ bool wait_count(const uint32_t* p, uint32_t target, uint32_t* err, uint64_t limit) {
  uint64_t t0 = 0;
  while (true) {
    uint32_t v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    if (v >= target) return true;
    const uint64_t now = globaltimer();
    if (t0 == 0) {
      t0 = now;
    } else if (now - t0 > limit) {
      raise_error(err, kErrTimeout);
      return false;
    }
    __nanosleep(64);
  }
}

// Selection of the min(K, pos+1) largest scores of every row this CTA holds
// part of, from the keys in shared memory (slot (item - it_lo) * 1024 + i =
// position 128 * tile_begin(item) + i).  All threads of the CTA take part.
//   1. rows of at most K candidates select every position;
//   2. the first digit's histogram of each row is summed over its CTAs and
//      gives the threshold bin b1 (like dsa_topk's first step);
//   3. fast path (the candidates fit one list per row): every CTA appends its
//      candidates (first digit >= b1) to the row's list, and the CTA holding
//      the row's last item resolves the other two digits in shared memory,
//      marks the selected positions (key > tau; key == tau, the lowest
//      positions first) in two bitmaps and writes them in ascending order;
//   4. otherwise every CTA of the row resolves digits two and three through
//      row histograms as well, then counts, per item, keys above and equal to
//      tau, and writes its own selections at the offsets those counts give.
// Rows meet at arrival counters (bounded waits).  A CTA takes its rows' steps
// in the order 2, 3 (publish), 4, 3 (resolve), so a CTA resolving a row never
// holds back a step another CTA waits on.
__device__ void fused_topk_tail(const IdxArgs& a, uint32_t* keys, int it_lo, int it_hi, TailSmem& sm) {
  using namespace topk;
  const int tid = threadIdx.x, nthreads = blockDim.x;
  const int4* recs = a.plan.items;
  const int K = a.K;
  const int nitems = it_hi - it_lo;  // <= kTailItemsMax (checked by the caller)
  if (tid < nitems) {
    const int4 ga = recs[2 * (it_lo + tid)], gb = recs[2 * (it_lo + tid) + 1];
    sm.item_info[tid] = make_int4(ga.y, ga.w, gb.x, gb.y);  // {token, position, tile begin, tile end}
  }
  __syncthreads();
  if (tid == 0) {
    int n = 0;
    for (int i = 0; i < nitems; ++i) {
      const int4 in = sm.item_info[i];
      if (n > 0 && sm.runs[n - 1].x == in.x)
        sm.runs[n - 1].z = it_lo + i + 1;
      else if (n < kTailRuns)
        sm.runs[n++] = make_int4(in.x, it_lo + i, it_lo + i + 1, in.y);
    }
    sm.nruns = n;
    sm.bad = 0;
  }
  __syncthreads();
  const int nruns = sm.nruns;
  auto info = [&](int item) { return sm.item_info[item - it_lo]; };
  auto run_s0 = [&](const int4& rn) { return 128 * info(rn.y).z; };  // first position of the run
  auto items_total = [&](int pos) { return (uint32_t)((((pos >> 7) + 1) + 7) >> 3); };
  auto holds_last = [&](const int4& rn) { return info(rn.z - 1).w == (rn.w >> 7) + 1; };
  auto arrive = [&](int token, int counter, uint32_t v) {  // after a __syncthreads
    if (tid == 0) {
      __threadfence();
      atomicAdd(a.tail + (int64_t)token * kTailWords + kTailArrive + counter, v);
    }
  };
  auto wait_row = [&](int token, int counter, int pos) {  // every CTA of the row arrived; ends with a barrier
    if (tid == 0 && !wait_count(a.tail + (int64_t)token * kTailWords + kTailArrive + counter, items_total(pos), a.err,
                                a.wait_ns))
      sm.bad = 1;
    __syncthreads();
    return !sm.bad;
  };
  auto load_hist = [&](const uint32_t* gh, int bins) {
    for (int b = tid; b < bins; b += nthreads) sm.hist[b] = __ldcg(gh + b);
    __syncthreads();
  };
  // 1. rows with at most K candidates: every candidate is selected, in order
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    const int pos = rn.w, n = pos + 1;
    if (n > K) continue;
    int32_t* out = a.idx + (int64_t)rn.x * K;
    const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024;
    for (int i = tid; i < L; i += nthreads)
      if (s0 + i <= pos) out[s0 + i] = s0 + i;
    if (holds_last(rn))  // the run holding the row's last tile pads it
      for (int s = n + tid; s < K; s += nthreads) out[s] = -1;
  }
  // 2. first digit: row histograms, then the threshold bin of each row
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K) continue;
    for (int b = tid; b < kD1Bins; b += nthreads) sm.hist[b] = 0u;
    __syncthreads();
    const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024;
    const uint32_t* kk = keys + (rn.y - it_lo) * 1024;
    for (int i = tid; i < L; i += nthreads)
      if (s0 + i <= rn.w) atomicAdd(&sm.hist[digit1(kk[i])], 1u);
    __syncthreads();
    uint32_t* gh = a.tail + (int64_t)rn.x * kTailWords;
    for (int b = tid; b < kD1Bins; b += nthreads)
      if (sm.hist[b]) atomicAdd(gh + b, sm.hist[b]);
    __syncthreads();
    arrive(rn.x, 0, (uint32_t)(rn.z - rn.y));
  }
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K) continue;
    if (!wait_row(rn.x, 0, rn.w)) return;
    load_hist(a.tail + (int64_t)rn.x * kTailWords, kD1Bins);
    find_bin<kD1Bins>(sm.hist, (uint32_t)K, &sm.bin, &sm.above);
    if (tid == 0) {
      const uint32_t nc = sm.above + sm.hist[sm.bin];
      sm.prefix[ri] = sm.bin;
      sm.need[ri] = (uint32_t)K - sm.above;
      sm.ncand[ri] = nc;
      sm.fast[ri] = nc <= (uint32_t)kCandCap && rn.w + 1 <= 32 * kBitmapWords;
    }
    __syncthreads();
  }
  // 3 (publish). fast rows: this CTA's candidates into the row's list
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K || !sm.fast[ri]) continue;
    const uint32_t b1 = sm.prefix[ri];
    const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024;
    const uint32_t* kk = keys + (rn.y - it_lo) * 1024;
    uint32_t cnt = 0;
    for (int i = tid; i < L; i += nthreads) cnt += (s0 + i <= rn.w && digit1(kk[i]) >= b1) ? 1u : 0u;
    if (tid < 2) sm.red[tid] = 0u;
    __syncthreads();
    cnt = __reduce_add_sync(0xffffffffu, cnt);
    if ((tid & 31) == 0) atomicAdd(&sm.red[0], cnt);
    __syncthreads();
    if (tid == 0) sm.red[2] = atomicAdd(a.tail + (int64_t)rn.x * kTailWords + kTailCandCount, sm.red[0]);
    __syncthreads();
    const uint32_t base = sm.red[2];
    int2* cl = a.cand + (int64_t)rn.x * kCandCap;
    for (int i = tid; i < L; i += nthreads) {
      const uint32_t key = kk[i];
      if (s0 + i <= rn.w && digit1(key) >= b1) {
        const uint32_t slot = base + atomicAdd(&sm.red[1], 1u);
        if (slot < (uint32_t)kCandCap) cl[slot] = make_int2(s0 + i, (int)key);
      }
    }
    __syncthreads();
    arrive(rn.x, 1, (uint32_t)(rn.z - rn.y));
  }
  // 4. other rows: digits two and three through row histograms, then counts
  for (int level = 1; level < 3 && !sm.bad; ++level) {
    const int bins = level < 2 ? kD1Bins : kD3Bins;
    for (int ri = 0; ri < nruns; ++ri) {
      const int4 rn = sm.runs[ri];
      if (rn.w + 1 <= K || sm.fast[ri]) continue;
      for (int b = tid; b < bins; b += nthreads) sm.hist[b] = 0u;
      __syncthreads();
      const uint32_t prefix = sm.prefix[ri];
      const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024;
      const uint32_t* kk = keys + (rn.y - it_lo) * 1024;
      for (int i = tid; i < L; i += nthreads) {
        if (s0 + i > rn.w) continue;
        const uint32_t key = kk[i];
        if (level == 1 ? digit1(key) == prefix : (key >> 10) == prefix)
          atomicAdd(&sm.hist[level == 1 ? digit2(key) : digit3(key)], 1u);
      }
      __syncthreads();
      uint32_t* gh = a.tail + (int64_t)rn.x * kTailWords + (level == 1 ? kD1Bins : 2 * kD1Bins);
      for (int b = tid; b < bins; b += nthreads)
        if (sm.hist[b]) atomicAdd(gh + b, sm.hist[b]);
      __syncthreads();
      arrive(rn.x, level, (uint32_t)(rn.z - rn.y));
    }
    for (int ri = 0; ri < nruns; ++ri) {
      const int4 rn = sm.runs[ri];
      if (rn.w + 1 <= K || sm.fast[ri]) continue;
      if (!wait_row(rn.x, level, rn.w)) return;
      load_hist(a.tail + (int64_t)rn.x * kTailWords + (level == 1 ? kD1Bins : 2 * kD1Bins), bins);
      if (level < 2)
        find_bin<kD1Bins>(sm.hist, sm.need[ri], &sm.bin, &sm.above);
      else
        find_bin<kD3Bins>(sm.hist, sm.need[ri], &sm.bin, &sm.above);
      if (tid == 0) {
        sm.prefix[ri] = (sm.prefix[ri] << (level < 2 ? 11 : 10)) | sm.bin;
        sm.need[ri] -= sm.above;
      }
      __syncthreads();
    }
  }
  if (sm.bad) return;
  // tau = the row's K-th largest key; need = how many tau-valued keys are taken
  // (the lowest positions).  Per run: keys above tau and equal to it.
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K || sm.fast[ri]) continue;
    const uint32_t tau = sm.prefix[ri];
    const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024;
    const uint32_t* kk = keys + (rn.y - it_lo) * 1024;
    uint32_t gt = 0, eq = 0;
    for (int i = tid; i < L; i += nthreads) {
      if (s0 + i > rn.w) continue;
      const uint32_t key = kk[i];
      gt += key > tau ? 1u : 0u;
      eq += key == tau ? 1u : 0u;
    }
    if (tid < 2) sm.red[tid] = 0u;
    __syncthreads();
    gt = __reduce_add_sync(0xffffffffu, gt);
    eq = __reduce_add_sync(0xffffffffu, eq);
    if ((tid & 31) == 0) {
      atomicAdd(&sm.red[0], gt);
      atomicAdd(&sm.red[1], eq);
    }
    __syncthreads();
    if (tid == 0) a.tail_items[rn.y] = make_int2((int)sm.red[0], (int)sm.red[1]);
    __syncthreads();
    arrive(rn.x, 3, (uint32_t)(rn.z - rn.y));
  }
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K || sm.fast[ri]) continue;
    if (tid < 2) sm.red[2 + tid] = 0u;
    if (!wait_row(rn.x, 3, rn.w)) return;
    // the row's selections in earlier items: counts of the runs before this one
    const int first = rn.y - (info(rn.y).z >> 3);  // the row's first item
    uint32_t bgt = 0, beq = 0;
    for (int k = first + tid; k < rn.y; k += nthreads) {
      const int2 c = __ldcg(a.tail_items + k);
      bgt += (uint32_t)c.x;
      beq += (uint32_t)c.y;
    }
    bgt = __reduce_add_sync(0xffffffffu, bgt);
    beq = __reduce_add_sync(0xffffffffu, beq);
    if ((tid & 31) == 0) {
      atomicAdd(&sm.red[2], bgt);
      atomicAdd(&sm.red[3], beq);
    }
    __syncthreads();
    const uint32_t tau = sm.prefix[ri], r = sm.need[ri];
    const uint32_t taken_eq = min(sm.red[3], r);
    const uint32_t off = sm.red[2] + taken_eq;
    const int s0 = run_s0(rn), L = (rn.z - rn.y) * 1024, pos = rn.w;
    const uint32_t* kk = keys + (rn.y - it_lo) * 1024;
    emit_selected(
        L, tau, r - taken_eq, K - (int)off,
        [&](int i) { return make_int2(s0 + i, s0 + i <= pos ? (int)kk[i] : 0); },
        a.idx + (int64_t)rn.x * K + off, sm.buf);
    __syncthreads();
  }
  // 3 (resolve). fast rows whose last item is here: the rest of the
  // selection from the row's candidate list, in shared memory (the score keys
  // are no longer needed: every step above that reads them is done)
  int2* cands = reinterpret_cast<int2*>(keys);
  uint32_t* gt_bits = reinterpret_cast<uint32_t*>(keys + 2 * kCandCap);
  uint32_t* eq_bits = gt_bits + kBitmapWords;
  for (int ri = 0; ri < nruns; ++ri) {
    const int4 rn = sm.runs[ri];
    if (rn.w + 1 <= K || !sm.fast[ri] || !holds_last(rn)) continue;
    if (!wait_row(rn.x, 1, rn.w)) return;
    const int nc = (int)sm.ncand[ri];
    const int2* cl = a.cand + (int64_t)rn.x * kCandCap;
    for (int i = tid; i < nc; i += nthreads) cands[i] = __ldcg(cl + i);
    const int nw = (rn.w + 32) >> 5;  // bitmap words of the row
    for (int w = tid; w < nw; w += nthreads) {
      gt_bits[w] = 0u;
      eq_bits[w] = 0u;
    }
    uint32_t prefix = sm.prefix[ri], need = sm.need[ri];
    for (int level = 1; level < 3; ++level) {  // digits two and three, over the candidates only
      const int bins = level < 2 ? kD1Bins : kD3Bins;
      for (int b = tid; b < bins; b += nthreads) sm.hist[b] = 0u;
      __syncthreads();
      for (int i = tid; i < nc; i += nthreads) {
        const uint32_t key = (uint32_t)cands[i].y;
        if (level == 1 ? digit1(key) == prefix : (key >> 10) == prefix)
          atomicAdd(&sm.hist[level == 1 ? digit2(key) : digit3(key)], 1u);
      }
      __syncthreads();
      if (level < 2)
        find_bin<kD1Bins>(sm.hist, need, &sm.bin, &sm.above);
      else
        find_bin<kD3Bins>(sm.hist, need, &sm.bin, &sm.above);
      prefix = (prefix << (level < 2 ? 11 : 10)) | sm.bin;
      need -= sm.above;
      __syncthreads();  // every thread has read bin / above
    }
    const uint32_t tau = prefix, r = need;  // r: tau-valued keys taken, the lowest positions first
    for (int i = tid; i < nc; i += nthreads) {
      const int2 c = cands[i];
      if ((uint32_t)c.y > tau)
        atomicOr(&gt_bits[c.x >> 5], 1u << (c.x & 31));
      else if ((uint32_t)c.y == tau)
        atomicOr(&eq_bits[c.x >> 5], 1u << (c.x & 31));
    }
    __syncthreads();
    // ascending emission: each thread takes a run of consecutive words
    const int per = (nw + nthreads - 1) / nthreads;
    const int w0 = min(nw, tid * per), w1 = min(nw, w0 + per);
    uint32_t my_gt = 0, my_eq = 0;
    for (int w = w0; w < w1; ++w) {
      my_gt += (uint32_t)__popc(gt_bits[w]);
      my_eq += (uint32_t)__popc(eq_bits[w]);
    }
    uint32_t tot;
    uint32_t gt_before = block_scan(my_gt, sm.buf, &tot);
    uint32_t eq_before = block_scan(my_eq, sm.buf, &tot);
    int32_t* out = a.idx + (int64_t)rn.x * K;
    for (int w = w0; w < w1; ++w) {
      uint32_t g = gt_bits[w], e = eq_bits[w];
      // eq bits of this word that are among the first r overall
      const uint32_t e_cnt = (uint32_t)__popc(e);
      if (eq_before >= r) {
        e = 0u;
      } else if (eq_before + e_cnt > r) {
        uint32_t keep = r - eq_before, m = 0u, x = e;
        while (keep--) {
          const uint32_t low = x & (~x + 1u);
          m |= low;
          x ^= low;
        }
        e = m;
      }
      eq_before += e_cnt;
      uint32_t sel = g | e;
      while (sel) {
        const int bit = __ffs(sel) - 1;
        sel &= sel - 1u;
        const uint32_t slot = gt_before + min(eq_before - e_cnt, r) + (uint32_t)__popc((g | e) & ((1u << bit) - 1u));
        if (slot < (uint32_t)K) out[slot] = (w << 5) + bit;
      }
      gt_before += (uint32_t)__popc(g);
    }
    __syncthreads();
  }
}

// Adds one epilogue warp's histogram of the current token to the global one
// and clears it (warp-private, so only the warp synchronises).
__device__ __forceinline__ void flush_hist(uint32_t* sh, uint32_t* gh, int t, int lane) {
  __syncwarp();
  for (int i = lane; i < kTopkHistBins; i += 32) {
    const uint32_t v = sh[i];
    if (v) {
      atomicAdd(gh + (int64_t)t * kTopkHistBins + i, v);
      sh[i] = 0u;
    }
  }
  __syncwarp();
}

template <bool kBf16, int TG, bool kFused, bool kMx>
__global__ void __launch_bounds__(kIdxThreads, 1)
k_index_scores_tc(const __grid_constant__ CUtensorMap tmap_k, const __grid_constant__ CUtensorMap tmap_q,
                  const IdxArgs a) {
  using C = IdxCfg<kBf16, TG, kFused, kMx>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* full = bars;                      // [NS]  stage loaded
  uint64_t* empty = bars + C::NS;             // [NS]  stage consumed (MMA + epilogue)
  uint64_t* b_full = bars + 2 * C::NS;        // [2]   group operands loaded
  uint64_t* b_empty = b_full + 2;             // [2]   group operands released
  uint64_t* acc_full = b_empty + 2;           // [NACC]
  uint64_t* acc_empty = acc_full + C::NACC;   // [NACC]
  uint64_t* mma_drain = acc_empty + C::NACC;  // every MMA this CTA issued has completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);
  const float* sc_smem = reinterpret_cast<const float*>(smem + C::OFF_SC);
  const float* w_smem = reinterpret_cast<const float*>(smem + C::OFF_W);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    // MXFP8: the producer's 32 lanes also arrive, once their scale copies land
    for (int i = 0; i < C::NS; ++i) {
      mbar_init(&full[i], kMx ? 1 + 32 : 1);
      mbar_init(&empty[i], 1 + 4);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&b_full[i], kMx ? 1 + 32 : 1);
      mbar_init(&b_empty[i], 1 + kEpiWarps);
    }
    for (int i = 0; i < C::NACC; ++i) {
      mbar_init(&acc_full[i], 1);
      mbar_init(&acc_empty[i], 4);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  pdl_wait();  // the plan and the quantized query come from the previous kernel
  pdl_trigger();

  // this CTA's contiguous share of the work items
  const int n_items = a.plan.counts[1];
  const int it_lo = (int)(((int64_t)n_items * blockIdx.x) / gridDim.x);
  const int it_hi = (int)(((int64_t)n_items * (blockIdx.x + 1)) / gridDim.x);

  const int4* recs = a.plan.items;  // item i: recs[2i] = {b, t0, cnt, pos0}, recs[2i+1] = {tile_begin, tile_end, g, 0}

  if (warp == 0) {
    // ------------------------------------------------------------ producer (whole warp)
    // Item records are fetched kRecAhead items ahead and each item's page ids
    // (one lane per page, <= 32 pages per item) kPgAhead items ahead, as
    // asynchronous copies into a ring in shared memory: one commit group per
    // item, so a page-table read has several items' worth of TMA issue to
    // hide behind.
    if (lane == 0) {
      prefetch_tmap(&tmap_k);
      prefetch_tmap(&tmap_q);
    }
    int4* ring_rec = reinterpret_cast<int4*>(smem + C::OFF_RING);                     // [slot][2]
    int* ring_pg = reinterpret_cast<int*>(smem + C::OFF_RING + kRingSlots * 32);     // [slot][32]
    auto issue_rec = [&](int it) {
      if (it < it_hi && lane < 2) cp_async_16(&ring_rec[(it % kRingSlots) * 2 + lane], recs + 2 * it + lane);
    };
    auto issue_pages = [&](int it) {  // the item's record is already in the ring
      if (it >= it_hi) return;
      const int4 ga = ring_rec[(it % kRingSlots) * 2], gb = ring_rec[(it % kRingSlots) * 2 + 1];
      const int lp = 2 * gb.x + lane;
      const int last = ga.w + ga.z - 1;
      if (lane < 2 * (gb.y - gb.x) && lp * kPage <= last)
        cp_async_4(&ring_pg[(it % kRingSlots) * 32 + lane], a.s.page_table + (int64_t)ga.x * a.s.max_pages + lp);
    };
    for (int i = 0; i < kRecAhead; ++i) issue_rec(it_lo + i);
    cp_async_commit();
    cp_async_wait<0>();
    __syncwarp();
    for (int i = 0; i < kPgAhead; ++i) {
      issue_pages(it_lo + i);
      cp_async_commit();
    }
    int stage = 0, sphase = 0, prev_g = -1, gcount = 0;
    int issued = 0, b_issued = 0;  // tiles / group operand loads with copies in flight or landed (lane 0)
    bool ok = true;
    for (int it = it_lo; it < it_hi && ok; ++it) {
      // groups so far: the page ids of it_lo .. it_lo+kPgAhead-1, then one
      // group per earlier iteration; all but the newest kPgAhead-1 hold what
      // this iteration reads (page ids of it, record of it+kPgAhead)
      cp_async_wait<kPgAhead - 1>();
      __syncwarp();
      issue_rec(it + kRecAhead);
      issue_pages(it + kPgAhead);
      cp_async_commit();
      const int4 ca = ring_rec[(it % kRingSlots) * 2], cb = ring_rec[(it % kRingSlots) * 2 + 1];
      const int pages = ring_pg[(it % kRingSlots) * 32 + lane];  // lanes past the item's pages are unused
      const int4 grp = ca;  // {b, t0, cnt, pos0}
      if (cb.z != prev_g) {
        const int slot = gcount & 1, use = gcount >> 1;
        int b_ok = 0;
        if (lane == 0) {
          if (!mbar_wait(&b_empty[slot], (use & 1) ^ 1, a.err, a.wait_ns)) {
            *abort_flag = 1;
          } else {
            b_ok = 1;
            const uint32_t wbytes = (uint32_t)grp.z * 256u;
            mbar_arrive_expect_tx(&b_full[slot], (uint32_t)C::B_BYTES + wbytes);
            uint8_t* bdst = smem + C::OFF_B + slot * C::B_BYTES;
            if constexpr (kBf16) {
              tma_load_2d(bdst, &tmap_q, &b_full[slot], 0, grp.y * 64);
              tma_load_2d(bdst + C::N * 128, &tmap_q, &b_full[slot], 64, grp.y * 64);
            } else {
              tma_load_2d(bdst, &tmap_q, &b_full[slot], 0, grp.y * 64);
            }
            bulk_load(smem + C::OFF_W + slot * TG * 256, a.w_operand + (int64_t)grp.y * 64, wbytes, &b_full[slot]);
            ++b_issued;
          }
        }
        if constexpr (kMx) {
          // the group's query scales: query row n = 64 k + h (token k, head h)
          // goes to row n % 32, column n / 32 of the scale-factor layout
          if (__shfl_sync(0xffffffffu, b_ok, 0)) {
            uint8_t* sfb = smem + C::OFF_SFB + slot * C::SFB_BYTES;
            for (int k = 0; k < grp.z; ++k)
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int col = 2 * k + c;
                cp_async_4(sfb + (col >> 2) * 512 + lane * 16 + (col & 3) * 4,
                           a.q_sf + ((int64_t)(grp.y + k) * 64 + 32 * c + lane) * 4);
              }
            cp_async_mbar_arrive(&b_full[slot]);  // once this lane's copies land
          }
        }
        prev_g = cb.z;
        ++gcount;
      }
      for (int tile = cb.x; tile < cb.y; ++tile) {
        const int j = tile - cb.x;
        const int pg0 = __shfl_sync(0xffffffffu, pages, 2 * j);
        const int pg1 = __shfl_sync(0xffffffffu, pages, 2 * j + 1);
        const int last = grp.w + grp.z - 1;
        int t_ok = 0;
        if (lane == 0 && !*abort_flag) {
          if (!mbar_wait(&empty[stage], sphase ^ 1, a.err, a.wait_ns)) {
            *abort_flag = 1;
          } else {
            t_ok = 1;
            int rows[2];
            const int pg[2] = {pg0, pg1};
            uint32_t bytes = 0;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              rows[h] = -1;
              if ((tile * 2 + h) * kPage <= last) {
                if (pg[h] >= 0 && pg[h] < a.s.num_phys_pages) {
                  rows[h] = pg[h] * kPage;
                  bytes += (uint32_t)(C::A_BYTES / 2) + ((kBf16 || kMx) ? 0u : 256u);
                } else {
                  raise_error(a.err, kErrBadIndex);
                }
              }
            }
            mbar_arrive_expect_tx(&full[stage], bytes);
            ++issued;
            uint8_t* adst = smem + C::OFF_A + stage * C::A_BYTES;
#pragma unroll
            for (int h = 0; h < 2; ++h) {
              if (rows[h] < 0) continue;
              if constexpr (kBf16) {
                tma_load_2d(adst + h * 8192, &tmap_k, &full[stage], 0, rows[h]);
                tma_load_2d(adst + 16384 + h * 8192, &tmap_k, &full[stage], 64, rows[h]);
              } else {
                tma_load_2d(adst + h * 8192, &tmap_k, &full[stage], 0, rows[h]);
                if constexpr (!kMx)
                  bulk_load(smem + C::OFF_SC + stage * 512 + h * 256, a.kI_scale + rows[h], 256, &full[stage]);
              }
            }
          }
        }
        if constexpr (kMx) {
          // the tile's key scales: key 32 c + l (page c / 2, row 32 (c % 2) + l)
          // goes to row l, column c; every lane arrives once its copies land
          if (__shfl_sync(0xffffffffu, t_ok, 0)) {
            uint8_t* sfa = smem + C::OFF_SC + stage * 512;
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const int h = c >> 1;
              const int pgh = h ? pg1 : pg0;
              if ((tile * 2 + h) * kPage <= last && pgh >= 0 && pgh < a.s.num_phys_pages)
                cp_async_4(sfa + lane * 16 + c * 4, a.kI_sf + ((int64_t)pgh * kPage + 32 * (c & 1) + lane) * 4);
            }
            cp_async_mbar_arrive(&full[stage]);
          }
        }
        if (++stage == C::NS) { stage = 0; sphase ^= 1; }
      }
      ok = __shfl_sync(0xffffffffu, (int)(*abort_flag == 0), 0) != 0;  // lane 0's view, warp-uniform
    }
    cp_async_wait<0>();  // no copy into the ring is still in flight at exit
    // drain, also after a failed wait: every copy this warp issued has landed
    // before the CTA exits (tile i used stage i % NS in phase i / NS; a stage's
    // last use is its only phase that can still be pending)
    if (lane == 0) {
      for (int i = issued > C::NS ? issued - C::NS : 0; i < issued; ++i)
        if (!mbar_wait(&full[i % C::NS], (uint32_t)((i / C::NS) & 1), a.err, kDrainLimitNs)) break;
      for (int i = b_issued > 2 ? b_issued - 2 : 0; i < b_issued; ++i)
        if (!mbar_wait(&b_full[i & 1], (uint32_t)((i >> 1) & 1), a.err, kDrainLimitNs)) break;
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------------ MMA issuer
      int stage = 0, sphase = 0, acc = 0, aphase = 0, prev_g = -1, gcount = 0, slot = 0;
      int4 nb = it_lo < it_hi ? recs[2 * it_lo + 1] : make_int4(0, 0, 0, 0);
      for (int it = it_lo; it < it_hi && !*abort_flag; ++it) {
        const int4 item = make_int4(nb.z, nb.x, nb.y, 0);  // {g, tile_begin, tile_end}
        if (it + 1 < it_hi) nb = recs[2 * it + 3];
        if (item.x != prev_g) {
          if (prev_g >= 0) mma_commit(&b_empty[slot]);  // previous group's operands free once its MMAs finish
          slot = gcount & 1;
          if (!mbar_wait(&b_full[slot], (gcount >> 1) & 1, a.err, a.wait_ns)) { *abort_flag = 1; break; }
          if constexpr (kMx) {  // the group's query scales into TMEM (in order before its MMAs)
            fence_proxy_async_smem();  // written by cp.async (generic proxy)
            tc_fence_after();
#pragma unroll
            for (int cp = 0; cp < C::SFB_COPIES; ++cp)
              tmem_cp_32x128b_x4(tmem + C::SFB0 + slot * C::SFB_COLS + 4 * cp,
                                 rows16_desc(smem_u32(smem + C::OFF_SFB + slot * C::SFB_BYTES + cp * 512)));
          }
          prev_g = item.x;
          ++gcount;
        }
        const uint32_t b_base = smem_u32(smem + C::OFF_B + slot * C::B_BYTES);
        for (int tile = item.y; tile < item.z; ++tile) {
          if (!mbar_wait(&full[stage], sphase, a.err, a.wait_ns)) { *abort_flag = 1; break; }
          if (!mbar_wait(&acc_empty[acc], aphase ^ 1, a.err, a.wait_ns)) { *abort_flag = 1; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + C::OFF_A + stage * C::A_BYTES);
          if constexpr (kMx) {
            // the tile's key scales into TMEM, then one block-scaled MMA per
            // 32-wide K block (byte k of each scale column)
            fence_proxy_async_smem();  // written by cp.async (generic proxy)
            tmem_cp_32x128b_x4(tmem + C::SFA0 + 4 * stage, rows16_desc(smem_u32(smem + C::OFF_SC + stage * 512)));
#pragma unroll
            for (int k = 0; k < 4; ++k)
              mma_mx(tmem + acc * C::N, sw128_kmajor_desc(a_base + k * 32), sw128_kmajor_desc(b_base + k * 32),
                     make_idesc_mx(128, C::N, k), (tmem + C::SFA0 + 4 * stage) | ((uint32_t)k << 30),
                     (tmem + C::SFB0 + slot * C::SFB_COLS) | ((uint32_t)k << 30), k > 0);
          } else {
#pragma unroll
            for (int k = 0; k < C::KSTEPS; ++k) {
              // K step k: 32 bytes inside a 128-byte swizzle row; bf16 rows span two 128-byte blocks
              const uint32_t a_off = kBf16 ? (k >> 2) * 16384 + (k & 3) * 32 : k * 32;
              const uint32_t b_off = kBf16 ? (k >> 2) * (C::N * 128) + (k & 3) * 32 : k * 32;
              mma_ss<kBf16>(tmem + acc * C::N, sw128_kmajor_desc(a_base + a_off), sw128_kmajor_desc(b_base + b_off),
                            C::IDESC, k > 0);
            }
          }
          mma_commit(&empty[stage]);
          mma_commit(&acc_full[acc]);
          if (++stage == C::NS) { stage = 0; sphase ^= 1; }
          if (++acc == C::NACC) { acc = 0; aphase ^= 1; }
        }
      }
      // drain, also after a failed wait: no MMA of this CTA still reads shared
      // memory or writes TMEM when the CTA deallocates and exits
      mma_commit(mma_drain);
      mbar_wait(mma_drain, 0, a.err, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------------ epilogue
    // Two warpgroups take alternate tiles (tile i -> warpgroup i & 1, which
    // therefore owns every other TMEM accumulator); both follow every group.
    const int q = (warp - 4) & 3;      // TMEM lane quarter of this warp
    const int wg = (warp - 4) >> 2;    // epilogue warpgroup
    const int r = q * 32 + lane;       // key row of the tile
    const uint32_t t_lane = tmem + ((uint32_t)(q * 32) << 16);
    int stage = 0, sphase = 0, acc = 0, aphase = 0, prev_g = -1, gcount = 0, slot = 0, prev_t = -1, ti = 0;
    float wreg[64];
    uint32_t* sh_hist = reinterpret_cast<uint32_t*>(smem + C::OFF_HIST) + (warp - 4) * kTopkHistBins;
    const bool do_hist = TG == 1 && !kFused && a.hist != nullptr;
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem + C::OFF_KEYS);
    if (do_hist) {
      for (int i = lane; i < kTopkHistBins; i += 32) sh_hist[i] = 0u;
      __syncwarp();
    }
    int4 na = make_int4(0, 0, 0, 0), nb = na;
    if (it_lo < it_hi) { na = recs[2 * it_lo]; nb = recs[2 * it_lo + 1]; }
    for (int it = it_lo; it < it_hi && !*abort_flag; ++it) {
      const int4 grp = na;                                // {b, t0, cnt, pos0}
      const int4 item = make_int4(nb.z, nb.x, nb.y, 0);  // {g, tile_begin, tile_end}
      if (it + 1 < it_hi) { na = recs[2 * it + 2]; nb = recs[2 * it + 3]; }
      if (item.x != prev_g) {
        if (prev_g >= 0) {
          __syncwarp();
          if (lane == 0) mbar_arrive(&b_empty[slot]);
        }
        if (do_hist && prev_t >= 0 && prev_t != grp.y) flush_hist(sh_hist, a.hist, prev_t, lane);
        prev_t = grp.y;
        slot = gcount & 1;
        if (!__all_sync(0xffffffffu, mbar_wait(&b_full[slot], (gcount >> 1) & 1, a.err, a.wait_ns))) {
          *abort_flag = 1;
          break;
        }
        if constexpr (TG == 1) {
#pragma unroll
          for (int h = 0; h < 64; ++h) wreg[h] = w_smem[slot * TG * 64 + h];
        }
        prev_g = item.x;
        ++gcount;
      }
      for (int tile = item.y; tile < item.z; ++tile, ++ti) {
        if ((ti & 1) == wg) {
          bool okw = mbar_wait(&acc_full[acc], aphase, a.err, a.wait_ns);
          // the row scales arrived with the stage's TMA; observe that completion here too
          if (!kBf16) okw = okw && mbar_wait(&full[stage], sphase, a.err, a.wait_ns);
          if (!__all_sync(0xffffffffu, okw)) { *abort_flag = 1; break; }
          tc_fence_after();
          const float sk = (kBf16 || kMx) ? 1.f : sc_smem[stage * 128 + r];
          __syncwarp();
          if (lane == 0) mbar_arrive(&empty[stage]);
          const int s = tile * 128 + r;
#pragma unroll 1
          for (int k = 0; k < TG; ++k) {
            uint32_t v0[32], v1[32];
            tmem_ld32(t_lane + acc * C::N + k * 64, v0);
            tmem_ld32(t_lane + acc * C::N + k * 64 + 32, v1);
            tmem_ld_wait_regs(v0);
            tmem_ld_wait_regs(v1);
            if (k == TG - 1) {  // every TMEM read of this accumulator is complete
              tc_fence_before();
              __syncwarp();
              if (lane == 0) mbar_arrive(&acc_empty[acc]);
            }
            const float* wk = w_smem + slot * TG * 64 + k * 64;
            float p0 = 0.f, p1 = 0.f, p2 = 0.f, p3 = 0.f;  // four chains instead of one
#pragma unroll
            for (int h = 0; h < 32; h += 2) {
              const float w0 = TG == 1 ? wreg[h] : wk[h];
              const float w1 = TG == 1 ? wreg[h + 1] : wk[h + 1];
              const float w2 = TG == 1 ? wreg[h + 32] : wk[h + 32];
              const float w3 = TG == 1 ? wreg[h + 33] : wk[h + 33];
              p0 = fmaf(w0, fmaxf(__uint_as_float(v0[h]), 0.f), p0);
              p1 = fmaf(w1, fmaxf(__uint_as_float(v0[h + 1]), 0.f), p1);
              p2 = fmaf(w2, fmaxf(__uint_as_float(v1[h]), 0.f), p2);
              p3 = fmaf(w3, fmaxf(__uint_as_float(v1[h + 1]), 0.f), p3);
            }
            const float score = ((p0 + p1) + (p2 + p3)) * sk;
            const bool valid = k < grp.z && s <= grp.w + k;
            if constexpr (kFused) {
              // the host sizes the grid so that a CTA's items fit; the guard keeps
              // an oversized share from writing past the buffer all the same
              if (it - it_lo < C::CAP_ITEMS) keys[(it - it_lo) * 1024 + (tile - item.y) * 128 + r] = order_key(score);
            } else {
              if (valid) a.scores[(int64_t)(grp.y + k) * a.ld + s] = score;
              // scores fall in random bins: a plain shared-memory add beats aggregating equal bins
              if (do_hist && valid) atomicAdd(&sh_hist[order_key(score) >> kTopkLowBits], 1u);
            }
          }
        }
        if (++stage == C::NS) { stage = 0; sphase ^= 1; }
        if (++acc == C::NACC) { acc = 0; aphase ^= 1; }
      }
    }
    __syncwarp();
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, C::TMEM_COLS);
  }
  if (TG == 1 && !kFused && a.hist != nullptr && !*abort_flag && it_hi > it_lo) {
    // the last token's histogram: the eight warps' copies summed here and
    // added once per CTA (earlier tokens were flushed per warp as they ended)
    const int t_last = recs[2 * (it_hi - 1)].y;
    const uint32_t* hb = reinterpret_cast<const uint32_t*>(smem + C::OFF_HIST);
    for (int i = threadIdx.x; i < kTopkHistBins; i += blockDim.x) {
      uint32_t v = 0;
#pragma unroll
      for (int w = 0; w < kEpiWarps; ++w) v += hb[w * kTopkHistBins + i];
      if (v) atomicAdd(a.hist + (int64_t)t_last * kTopkHistBins + i, v);
    }
  }
  if constexpr (kFused) {
    // the selection, once every score of this CTA is in shared memory (the
    // barrier above); a CTA that gave up on a wait leaves its rows to time out
    if (!*abort_flag && it_hi - it_lo <= C::CAP_ITEMS)
      fused_topk_tail(a, reinterpret_cast<uint32_t*>(smem + C::OFF_KEYS), it_lo, it_hi,
                      *reinterpret_cast<TailSmem*>(smem + C::OFF_TAIL));
  }
}

// ---------------------------------------------------------------- host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

// Row-major 2-D map: rows of `row_elems` elements, box of box_x x box_y, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, bool bf16, uint64_t row_elems, uint64_t rows, uint32_t box_x,
              uint32_t box_y) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {row_elems, rows};
  const cuuint64_t strides[1] = {row_elems * (bf16 ? 2 : 1)};
  const cuuint32_t box[2] = {box_x, box_y};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base),
            dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count() {
  int dev = 0, n = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n > 0 ? n : 148;
}

template <bool kBf16, int TG, bool kFused, bool kMx = false>
cudaError_t launch_tc(const CUtensorMap& mk, const CUtensorMap& mq, const IdxArgs& a, int grid, cudaStream_t st) {
  using C = IdxCfg<kBf16, TG, kFused, kMx>;
  static thread_local int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(k_index_scores_tc<kBf16, TG, kFused, kMx>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, C::SMEM);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  cudaError_t e = launch_pdl("index_scores", k_index_scores_tc<kBf16, TG, kFused, kMx>, dim3(grid), dim3(kIdxThreads),
                             (size_t)C::SMEM, st, mk, mq, a);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace

int indexer_fused_capacity() {
  const int a = IdxCfg<false, 1, true>::CAP_ITEMS, b = IdxCfg<true, 1, true>::CAP_ITEMS;
  const int c = IdxCfg<false, 1, true, true>::CAP_ITEMS;
  const int ab = a < b ? a : b;
  return ab < c ? ab : c;
}

bool indexer_fused_fits(int T, int B, int max_ctx) {
  if (T != B) return false;  // one query token per sequence
  const int64_t items = plan_max_items(T, B, max_ctx, 1);
  return (items + kFusedGrid - 1) / kFusedGrid <= indexer_fused_capacity();
}

int64_t fused_topk_words(int T, int B, int max_ctx) {
  return (int64_t)T * kTailWords + 2 * plan_max_items(T, B, max_ctx, 1);
}

size_t fused_topk_cand_bytes(int T) { return (size_t)T * kCandCap * sizeof(int2); }

cudaError_t launch_index_scores(const SeqsDev& s, const PlanBufs& plan, int tg, const void* q_operand,
                                const float* w_operand, const uint8_t* q_sf, const void* kI, const void* kI_scale,
                                IdxFmt fmt, float* scores, int64_t ld, uint32_t* hist, uint32_t* err,
                                cudaStream_t st, const FusedTopk* fused) {
  const bool bf16 = fmt == IdxFmt::kBf16, mx = fmt == IdxFmt::kMx;
  const uint64_t R = (uint64_t)s.num_phys_pages * kPage;
  const uint64_t qrows = (uint64_t)s.num_tokens * kHI;
  CUtensorMap mk, mq;
  if (!make_map(&mk, kI, bf16, kDI, R, bf16 ? 64 : 128, 64)) return cudaErrorInvalidValue;
  if (!make_map(&mq, q_operand, bf16, kDI, qrows, bf16 ? 64 : 128, 64 * tg)) return cudaErrorInvalidValue;
  IdxArgs a{s,
            plan,
            w_operand,
            fmt == IdxFmt::kE4M3 ? static_cast<const float*>(kI_scale) : nullptr,
            mx ? static_cast<const uint8_t*>(kI_scale) : nullptr,
            mx ? q_sf : nullptr,
            scores,
            ld,
            tg == 1 ? hist : nullptr,
            err,
            wait_limit_ns(),
            fused ? fused->tail : nullptr,
            fused ? fused->tail_items : nullptr,
            fused ? fused->cand : nullptr,
            fused ? fused->idx : nullptr,
            fused ? fused->K : 0};
  const int grid = sm_count();
  if (fused) {
    // the rows' CTAs wait on one another: every CTA must be resident (one per
    // SM) and hold at most the capacity the workspace was sized for
    if (tg != 1 || grid < kFusedGrid) return cudaErrorInvalidConfiguration;
    if (mx) return launch_tc<false, 1, true, true>(mk, mq, a, kFusedGrid, st);
    return bf16 ? launch_tc<true, 1, true>(mk, mq, a, kFusedGrid, st) : launch_tc<false, 1, true>(mk, mq, a, kFusedGrid, st);
  }
  if (mx) {
    if (tg == 1) return launch_tc<false, 1, false, true>(mk, mq, a, grid, st);
    if (tg == 2) return launch_tc<false, 2, false, true>(mk, mq, a, grid, st);
  } else if (!bf16) {
    if (tg == 1) return launch_tc<false, 1, false>(mk, mq, a, grid, st);
    if (tg == 4) return launch_tc<false, 4, false>(mk, mq, a, grid, st);
  } else {
    if (tg == 1) return launch_tc<true, 1, false>(mk, mq, a, grid, st);
    if (tg == 2) return launch_tc<true, 2, false>(mk, mq, a, grid, st);
  }
  return cudaErrorInvalidValue;
}

}  // namespace dsa
