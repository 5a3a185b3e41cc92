// Sparse MLA attention over the selected latent rows, on the 5th-generation
// tensor cores ([P1] "Day 0 Inference Adaptation and Performance Optimization
// for Hybrid Attention LLMs", Understanding the New Architecture item 2;
// [P2] "Hybrid Attention LLM Inference Acceleration...", section 2 item 2
// "Sparse attention computation"; [P5] "Day-0 Inference Adaptation for Large
// Language Models...", Operator Fusion and Memory Access Optimization,
// bullet 1: the Top-K indices go straight into the compute kernel, which
// gathers the rows itself -- no gathered KV copy exists):
//
//   out[t,h,:] = sum_{s in idx[t]} p_s KV[s,0:512],
//   p = softmax_s(scale * q[t,h,:] . KV[s,0:576]),   lse = ln sum exp(...)
//
// The fp32 accumulator of 128 heads x 512 value dims fills all of TMEM, so
// the work of one (token, slice of the index list) goes to a CLUSTER OF TWO
// CTAs.  CTA r owns value dims [256r, 256r+256) and the key dims
// {256r..256r+255} u {512+32r..512+32r+31}; it gathers only those 576 bytes of
// each selected row.  Three warps resolve every selected row of the slice
// up front (index list -> page table, all loads independent) and then copy
// the rows block by block with 16-byte cp.async straight into the 128-byte /
// 64-byte swizzled operand layouts -- many small copies in flight instead of
// a queue of four-row TMA gathers.  Per block of 64 selected rows:
//   * S_r = Q_r K_r^T (M = 128 heads, N = 64 rows, K = 288 dims) into TMEM;
//   * the two partial S are exchanged through distributed shared memory
//     (st.async into the peer's double-buffered receive area, counted on the
//     peer's mbarrier, so no cluster-scope fence sits on the path) and summed
//     (a + b = b + a, so both CTAs hold bit-identical logits and take
//     identical softmax decisions);
//   * online softmax in registers (one head row per thread, base-2 exponent,
//     the running maximum is only moved -- and O rescaled in TMEM -- when it
//     grows by more than 2^8, which is exact because O and l share it);
//   * P goes to TMEM as two bf16 terms, P = P_hi + P_lo (together within
//     2^-17 of the fp32 value; one bf16 term alone would leave a relative
//     error of 2^-9 on rows dominated by a few selected keys), and
//     O_r += P_hi V_r + P_lo V_r (M = 128, N = 256, K = 64) accumulates in
//     TMEM with P read from TMEM, V_r being the same gathered bytes read as an
//     MN-major operand.  TMEM columns: O [0, 256), S [256, 384) (two
//     buffers), P [384, 512) (two buffers of hi + lo).
// Slices of one token are merged by k_combine (log-sum-exp weights).
#include <cudaTypedefs.h>

#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kBK = 64;                      // selected rows per block
constexpr int kQLatBytes = 128 * 128;        // one 64-dim swizzle atom of 128 head rows
constexpr int kQBytes = 4 * kQLatBytes + 128 * 64;
constexpr int kKVStage = 4 * kBK * 128 + kBK * 64;  // 36864: 4 latent atoms + rope quarter
constexpr int kXBytes = 128 * kBK * 4;       // one partial S: [16 column quads][128 heads][4] fp32
constexpr int kLoaders = 96;                 // warps 0, 2, 3 copy the selected rows
constexpr int kRingBlocks = kMaxK / kBK;     // resolved row ids of every block of a slice
constexpr int kLoaderBarrier = 1;            // named barrier of the loader warps
constexpr int OFF_Q = 0;
constexpr int OFF_KV = OFF_Q + kQBytes;                 // 73728
constexpr int kStages = 3;                              // row stages in flight
constexpr int OFF_X = OFF_KV + kStages * kKVStage;      // 184320: the peer's partial logits
constexpr int OFF_ROWS = OFF_X + kXBytes;               // 217088: [block][64] pool rows (-1 = masked)
constexpr int OFF_MASK = OFF_ROWS + kRingBlocks * kBK * 4;  // [block] 64-bit validity masks
constexpr int OFF_BAR = OFF_MASK + kRingBlocks * 8;
constexpr int kNBars = 17;
constexpr int OFF_PAIR = OFF_BAR + kNBars * 8;          // [2 parity][2 half][128 heads] float2
constexpr int OFF_MISC = OFF_PAIR + 2 * 2 * 128 * 8;
constexpr int SMEM_BYTES = OFF_MISC + 16 + 1024;
constexpr int kThreads = 384;                // warps 0, 2, 3 load; 1 issues MMAs; 4-11 softmax
constexpr int kPairBarrier = 2;              // named barriers 2..5: softmax warps w and w+4
static_assert(SMEM_BYTES <= 227 * 1024, "shared memory");
static_assert(OFF_KV % 1024 == 0 && kKVStage % 1024 == 0, "swizzle atoms need 1024-B alignment");
constexpr uint32_t kTmemS = 256, kTmemP = 384;  // TMEM column bases (O at 0)

constexpr uint32_t IDESC_QK = make_idesc_major(true, 128, kBK, 0, 0);  // S = Q K^T, both K-major
constexpr uint32_t IDESC_PV = make_idesc_major(true, 128, 256, 0, 1);  // O += P V, V MN-major
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;    // log2 units

// 2^x from the MUFU unit (approximate, subnormal results flushed to 0;
// ex2(-inf) = +0).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void store_out(void* out, bool f32, int64_t i, float v) {
  if (f32)
    reinterpret_cast<float*>(out)[i] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16(v);
}

struct AttnArgs {
  SeqsDev s;
  TokenMap tm;
  const __nv_bfloat16* kv;  // latent pool [rows, 576]
  const int32_t* idx;
  int K, H, ks, splits;
  bool tm_early;     // the token map was written two or more launches back
  float scale_log2;  // scale * log2(e)
  void* out;
  bool out_f32;
  float* lse;
  float* part_o;
  float2* part_ml;
  uint32_t* err;
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
k_sparse_mla_tc(const __grid_constant__ CUtensorMap tq_lat, const __grid_constant__ CUtensorMap tq_rope,
                const AttnArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + OFF_BAR);
  uint64_t* q_full = bars + 0;
  uint64_t* kv_full = bars + 1;    // [kStages] rows of block j (stage j % 3) landed
  uint64_t* kv_empty = bars + 4;   // [kStages] PV of the stage's block completed
  uint64_t* s_full = bars + 7;     // [2] S of block j (buffer j & 1) in TMEM
  uint64_t* s_empty = bars + 9;    // [2] S buffer read by every softmax warp
  uint64_t* p_full = bars + 11;    // [2] P of block j (buffer j & 1) in TMEM
  uint64_t* o_done = bars + 13;    // [2] PV of block i (buffer i & 1) has completed
  uint64_t* x_full = bars + 15;    // the peer's partial S of the current block has landed in X
  uint64_t* x_free = bars + 16;    // the peer's eight softmax warps have read what I sent
  int32_t* ring_rows = reinterpret_cast<int32_t*>(smem + OFF_ROWS);
  uint64_t* ring_mask = reinterpret_cast<uint64_t*>(smem + OFF_MASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const uint32_t peer = rank ^ 1u;
  const int cluster = blockIdx.x >> 1;
  const int t = cluster / a.splits, sp = cluster % a.splits;
  const int kbeg = sp * a.ks;
  const int kend = min(a.K, kbeg + a.ks);

  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], kLoaders + 1);  // every loader's copies + the mask's publisher
      mbar_init(&kv_empty[i], 1);
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_empty[i], 8);
      mbar_init(&p_full[i], 8);  // one arrival per softmax warp
      mbar_init(&o_done[i], 1);
    }
    mbar_init(x_full, 1);   // armed by this CTA (expect_tx), filled by the peer's st.async
    mbar_init(x_free, 8);   // one arrival per peer softmax warp
    *abort_flag = 0;
    fence_mbar_init();
    // the receive area for block 0 is armed before the cluster barrier below
    // lets the peer store into it
    mbar_arrive_expect_tx(x_full, kXBytes);
  }
  if (warp == 2) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any remote arrive
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {  // q is an input of the call: its load overlaps the wait below
    prefetch_tmap(&tq_lat);
    mbar_arrive_expect_tx(q_full, kQBytes);
    for (int at = 0; at < 4; ++at)
      tma_load_2d(smem + OFF_Q + at * kQLatBytes, &tq_lat, q_full, 256 * rank + 64 * at, t * a.H);
    tma_load_2d(smem + OFF_Q + 4 * kQLatBytes, &tq_rope, q_full, 512 + 32 * rank, t * a.H);
  }
  // the token map can be read before the wait when it does not come from
  // the kernel just before; the index lists always do
  int pos = a.tm_early ? a.tm.pos[t] : 0, b = a.tm_early ? a.tm.seq[t] : 0;
  if (a.tm_early && warp == 0 && pos >= 0) {
    // the sequence's page-table row into L2 while the previous kernel ends:
    // the loaders look selected pages up in it right after the wait
    const int64_t row_bytes = (int64_t)a.s.max_pages * 4;
    const char* pt = reinterpret_cast<const char*>(a.s.page_table + (int64_t)b * a.s.max_pages);
    for (int64_t off = (int64_t)lane * 128; off < row_bytes; off += 32 * 128) prefetch_l2(pt + off);
  }
  pdl_wait();
  pdl_trigger();
  if (!a.tm_early) {
    pos = a.tm.pos[t];
    b = a.tm.seq[t];
  }
  const int nblk = (pos >= 0 && kend > kbeg) ? (kend - kbeg + kBK - 1) / kBK : 0;

  if ((warp == 0 || warp == 2 || warp == 3) && nblk > 0) {
    // ---------------------------------------------------------------- loaders
    const int li = (warp == 0 ? 0 : warp - 1) * 32 + lane;  // 0 .. 95
    const int lw = warp == 0 ? 0 : warp - 1;                // loader warp 0 .. 2
    // Pool rows of every block of the slice, resolved up front in three
    // passes whose loads are all independent: the index list, then the page
    // ids (both staged by cp.async in the KV stage areas, which the first row
    // copies overwrite only after the last pass), then rows and masks
    // (row -1 = masked).
    {
      const int nkeys = kend - kbeg;
      int32_t* s_sidx = reinterpret_cast<int32_t*>(smem + OFF_KV);
      int32_t* s_page = reinterpret_cast<int32_t*>(smem + OFF_KV + kKVStage);
      const int32_t* idx_row = a.idx + (int64_t)t * a.K + kbeg;
      for (int k = li; k < nkeys; k += kLoaders) cp_async_4(&s_sidx[k], idx_row + k);
      cp_async_wait_all();
      bar_red_or(kLoaderBarrier, kLoaders, false);
      const int32_t* pt_row = a.s.page_table + (int64_t)b * a.s.max_pages;
      for (int k = li; k < nkeys; k += kLoaders) {
        const int sidx = s_sidx[k];
        if (sidx >= 0 && sidx <= pos) cp_async_4(&s_page[k], pt_row + (sidx >> 6));  // sidx <= pos: inside the table
      }
      cp_async_wait_all();
      bar_red_or(kLoaderBarrier, kLoaders, false);
      for (int k = li; k < nblk * kBK; k += kLoaders) {
        int row = -1;
        if (k < nkeys) {
          const int sidx = s_sidx[k];
          if (sidx >= 0 && sidx <= pos) {
            const int page = s_page[k];
            if (page >= 0 && page < a.s.num_phys_pages)
              row = page * kPage + (sidx & (kPage - 1));
            else
              raise_error(a.err, kErrBadIndex);
          } else if (sidx != -1) {
            raise_error(a.err, kErrBadIndex);
          }
        }
        ring_rows[k] = row;
      }
      bar_red_or(kLoaderBarrier, kLoaders, false);
      for (int w32 = lw; w32 < 2 * nblk; w32 += 3) {  // 32 rows per warp -> half a block's mask
        const uint32_t m = __ballot_sync(0xffffffffu, ring_rows[w32 * 32 + lane] >= 0);
        if (lane == 0) reinterpret_cast<uint32_t*>(ring_mask)[w32] = m;
      }
    }
    const uint32_t kv_smem = smem_u32(smem + OFF_KV);
    const __nv_bfloat16* kv_base = reinterpret_cast<const __nv_bfloat16*>(a.kv);
    bool failed = bar_red_or(kLoaderBarrier, kLoaders, false);
    for (int j = 0; j < nblk && !failed; ++j) {
      const int stage = j % kStages, slot = j;
      bool ok = mbar_wait(&kv_empty[stage], ((j / kStages) & 1) ^ 1, a.err);
      if (ok) {
        // one warp per row: lane k copies latent piece k (16 B = 8 dims) of
        // the CTA's 256 latent dims; rope pieces go 8 rows per instruction
        const uint32_t dst0 = kv_smem + stage * kKVStage;
        for (int r = lw; r < kBK; r += 3) {
          const int row = ring_rows[slot * kBK + r];
          const bool v = row >= 0;
          const uint32_t dst = dst0 + (lane >> 3) * (kBK * 128) + r * 128 +
                               ((((uint32_t)lane & 7u) ^ ((uint32_t)r & 7u)) << 4);
          cp_async_16_zfill(dst, kv_base + (v ? (int64_t)row * kDQK + 256 * rank + 8 * lane : 0), v ? 16u : 0u);
        }
        for (int g8 = lw; g8 < kBK / 8; g8 += 3) {
          const int r = 8 * g8 + (lane >> 2);
          const uint32_t kr = (uint32_t)lane & 3u;
          const int row = ring_rows[slot * kBK + r];
          const bool v = row >= 0;
          const uint32_t dst = dst0 + 4 * (kBK * 128) + r * 64 + ((kr ^ (((uint32_t)r >> 1) & 3u)) << 4);
          cp_async_16_zfill(dst, kv_base + (v ? (int64_t)row * kDQK + 512 + 32 * rank + 8 * kr : 0), v ? 16u : 0u);
        }
      }
      cp_async_mbar_arrive(&kv_full[stage]);  // counts once this thread's copies land
      if (li == 0) mbar_arrive(&kv_full[stage]);  // releases the masks read by the softmax warps
      failed = bar_red_or(kLoaderBarrier, kLoaders, !ok);
      if (failed) *abort_flag = 1;
    }
    cp_async_wait_all();
    // drain: every stage has been consumed by the MMA before the CTA exits
    if (li == 0 && !*abort_flag) {
      for (int j = nblk; j < nblk + kStages; ++j)
        if (!mbar_wait(&kv_empty[j % kStages], ((j / kStages) & 1) ^ 1, a.err)) break;
    }
    __syncwarp();
  } else if (warp == 1 && nblk > 0) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t q_base = smem_u32(smem + OFF_Q);
      const uint32_t kv_base = smem_u32(smem + OFF_KV);
      bool ok = mbar_wait(q_full, 0, a.err);
      // Issue whichever is ready, PV first (it frees a row stage):
      //   PV(i) once P(i) is in TMEM;
      //   QK(j) once block j's rows have landed, S buffer j & 1 is free and
      //   PV(j-2) has been issued -- so s_full(j), which tracks every earlier
      //   MMA, also tells the softmax warps that P buffer j & 1 is free.
      int nq = 0, np = 0;  // next block to score / to accumulate
      uint64_t idle_since = 0;
      while (ok && np < nblk) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        if (np < nq && mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) {
          tc_fence_after();
          const uint32_t vb = kv_base + (np % kStages) * kKVStage;
          const uint32_t pb = tmem + kTmemP + 64 * (np & 1);  // P_hi at +0, P_lo at +32 (16 keys per 8 columns)
#pragma unroll
          for (int term = 0; term < 2; ++term)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ts_bf16(tmem, pb + 32 * term + 8 * kk, smem_desc(vb + kk * 2048, 8192, 1024, 2), IDESC_PV,
                          np > 0 || term > 0 || kk > 0);
          mma_commit(&kv_empty[np % kStages]);
          mma_commit(&o_done[np & 1]);
          ++np;
          idle_since = 0;
        } else if (nq < nblk && nq < np + 2 && mbar_test_wait(&kv_full[nq % kStages], (nq / kStages) & 1) &&
                   mbar_test_wait(&s_empty[nq & 1], ((nq >> 1) & 1) ^ 1)) {
          fence_proxy_async_smem();  // the rows were written by cp.async (generic proxy)
          tc_fence_after();
          const uint32_t d = tmem + kTmemS + kBK * (nq & 1);
          const uint32_t kb = kv_base + (nq % kStages) * kKVStage;
#pragma unroll
          for (int at = 0; at < 4; ++at)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              mma_ss<true>(d, smem_desc(q_base + at * kQLatBytes + kk * 32, 16, 1024, 2),
                           smem_desc(kb + at * (kBK * 128) + kk * 32, 16, 1024, 2), IDESC_QK, (at | kk) != 0);
#pragma unroll
          for (int kk = 0; kk < 2; ++kk)
            mma_ss<true>(d, smem_desc(q_base + 4 * kQLatBytes + kk * 32, 16, 512, 4),
                         smem_desc(kb + 4 * (kBK * 128) + kk * 32, 16, 512, 4), IDESC_QK, true);
          mma_commit(&s_full[nq & 1]);
          ++nq;
          idle_since = 0;
        } else {
          const uint64_t now = globaltimer();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > kWaitLimitNs) {
            raise_error(a.err, kErrTimeout);
            ok = false;
          }
          __nanosleep(32);
        }
      }
      if (!ok) *abort_flag = 1;
    }
    __syncwarp();
  } else if (warp >= 4 && nblk > 0) {
    // ---------------------------------------------------------------- softmax / exchange / epilogue
    // Eight warps: warp 4+q and warp 8+q share TMEM lane quarter q (heads
    // 32q .. 32q+31); half g = 0 / 1 takes logits 32g .. 32g+31 of every
    // block and value dims 128g .. 128g+127 of O.  The two halves of a head
    // combine their maxima (and at the end their sums) through shared memory
    // at a 64-thread named barrier, which also carries any failure, so both
    // warps of a pair always leave together.
    const int sw = warp - 4, half = sw >> 2, qw = sw & 3;
    const int h = qw * 32 + lane;  // head row = TMEM lane
    const int cb = 32 * half;      // this half's first logit of a block
    const uint32_t t_lane = tmem + ((uint32_t)(qw * 32) << 16);
    const int pair_bar = kPairBarrier + qw;
    float2* pair = reinterpret_cast<float2*>(smem + OFF_PAIR);  // [parity][half][head]
    // X[b][c][h] holds logits 4c .. 4c+3 of head h: a warp's stores of one c
    // are 512 contiguous bytes
    const float4* xcol = reinterpret_cast<const float4*>(smem + OFF_X) + h;
    const uint32_t x_peer = map_peer(smem_u32(smem + OFF_X), peer) + (uint32_t)h * 16u;
    const uint32_t x_full_peer = map_peer(smem_u32(x_full), peer);
    const uint32_t x_free_peer = map_peer(smem_u32(x_free), peer);
    const float sc = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;  // l: this half's share of the sum
    bool good = true;
    for (int j = 0; j < nblk; ++j) {
      const int sb = j & 1;
      // s_full(j) also means PV(j-2) is complete (it was issued before QK(j)),
      // so P's buffer sb is free
      good = good && __all_sync(0xffffffffu, !*abort_flag && mbar_wait(&s_full[sb], (j >> 1) & 1, a.err));
      uint32_t v[32];
      if (good) {
        tc_fence_after();
        tmem_ld32(t_lane + kTmemS + kBK * sb + cb, v);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&s_empty[sb]);
      }
      // the peer's warps have read my previous block: its receive area is free
      if (j >= 1) good = good && __all_sync(0xffffffffu, mbar_wait_cluster(x_free, (j - 1) & 1, a.err));
      if (good) {
        // my partial logits -> the peer's receive area, counted on its x_full
#pragma unroll
        for (int c = 0; c < 8; ++c)
          st_async_v4(x_peer + (8 * half + c) * 2048, v[4 * c], v[4 * c + 1], v[4 * c + 2], v[4 * c + 3],
                      x_full_peer);
      }
      good = good && __all_sync(0xffffffffu, mbar_wait_cluster(x_full, j & 1, a.err));
      float s[32];
      if (good) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
          const float4 pv4 = xcol[(8 * half + c) * 128];
          s[4 * c + 0] = __uint_as_float(v[4 * c]) + pv4.x;
          s[4 * c + 1] = __uint_as_float(v[4 * c + 1]) + pv4.y;
          s[4 * c + 2] = __uint_as_float(v[4 * c + 2]) + pv4.z;
          s[4 * c + 3] = __uint_as_float(v[4 * c + 3]) + pv4.w;
        }
        // re-arm my receive area for block j+1, then tell the peer this
        // warp is done with it: the peer stores block j+1 only after all
        // eight signals, the re-arming warp's among them
        if (sw == 0 && lane == 0 && j + 1 < nblk) mbar_arrive_expect_tx(x_full, kXBytes);
        __syncwarp();  // every lane's reads of X precede the signal
        if (lane == 0) mbar_arrive_remote_relaxed(x_free_peer);
      }
      // validity of the block's rows (published before the stage completed)
      good = good && __all_sync(0xffffffffu, mbar_wait(&kv_full[j % kStages], (j / kStages) & 1, a.err));
      float mraw = -INFINITY, mneg = INFINITY;
      if (good) {
        const uint32_t m32 = (uint32_t)(ring_mask[j] >> cb);
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          const bool on = (m32 >> i) & 1u;
          s[i] = on ? s[i] : -INFINITY;
          mraw = fmaxf(mraw, s[i]);
          mneg = fminf(mneg, on ? s[i] : INFINITY);
        }
        pair[((j & 1) * 2 + half) * 128 + h] = make_float2(mraw, mneg);
      }
      if (bar_red_or(pair_bar, 64, !good)) {  // either half failed: both leave
        good = false;
        break;
      }
      const float2 other = pair[((j & 1) * 2 + (half ^ 1)) * 128 + h];
      mraw = fmaxf(mraw, other.x);
      mneg = fminf(mneg, other.y);
      // scale <= 0 (allowed, if odd): the largest scaled logit comes from the smallest raw one
      const float mblk = mraw == -INFINITY ? -INFINITY : (sc > 0.f ? mraw * sc : mneg * sc);
      const bool move = mblk > m_ref + kRescaleThreshold;
      const float m_new = move ? mblk : m_ref;
      const float alpha = move ? exp2f(m_ref - m_new) : 1.f;  // exp2(-inf) = 0 on the first block
      const float mu = m_new == -INFINITY ? 0.f : m_new;      // nothing unmasked yet: every term is 0
      uint32_t pk[16], pl[16];
      float psum = 0.f;
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // masked: s = -inf and sc > 0 give ex2(-inf) = 0; sc <= 0 takes the select
        const float x0 = fmaf(s[2 * i], sc, -mu), x1 = fmaf(s[2 * i + 1], sc, -mu);
        const float e0 = sc > 0.f ? ex2_ftz(x0) : (s[2 * i] == -INFINITY ? 0.f : ex2_ftz(x0));
        const float e1 = sc > 0.f ? ex2_ftz(x1) : (s[2 * i + 1] == -INFINITY ? 0.f : ex2_ftz(x1));
        psum += e0 + e1;
        const __nv_bfloat162 hi = __floats2bfloat162_rn(e0, e1);
        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hi);
        const __nv_bfloat162 lo =
            __floats2bfloat162_rn(e0 - __uint_as_float(hb << 16), e1 - __uint_as_float(hb & 0xFFFF0000u));
        pk[i] = hb;
        pl[i] = *reinterpret_cast<const uint32_t*>(&lo);
      }
      // P_hi: columns kTmemP + 64 sb + [0, 32), P_lo: + [32, 64); 16 columns per half
      tmem_st16(t_lane + kTmemP + 64 * sb + 16 * half, pk);
      tmem_st16(t_lane + kTmemP + 64 * sb + 32 + 16 * half, pl);
      // TMEM loads/stores are warp-wide: if any head of the warp moved its
      // maximum, the warp rescales its half of O (alpha = 1 leaves a row
      // exact), once PV(j-1) -- the last writer of O -- has completed
      if (j >= 1 && __any_sync(0xffffffffu, move && m_ref != -INFINITY)) {
        good = __all_sync(0xffffffffu, mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err));
        if (good) {
          tc_fence_after();
#pragma unroll 1
          for (int c = 0; c < 4; ++c) {
            uint32_t o[32];
            tmem_ld32(t_lane + 128 * half + 32 * c, o);
            tmem_ld_wait();
#pragma unroll
            for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
            tmem_st32(t_lane + 128 * half + 32 * c, o);
          }
        }
      }
      l = l * alpha + psum;
      m_ref = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (good && lane == 0) mbar_arrive(&p_full[sb]);
    }
    // epilogue: O / l for this half's 128 value dims.  tcgen05.ld is
    // warp-wide, so a warp with any valid head loads; only the stores test h < H.
    good = good && __all_sync(0xffffffffu, mbar_wait(&o_done[(nblk - 1) & 1], ((nblk - 1) >> 1) & 1, a.err));
    // the sums go through the parity the last block did not use: its maxima
    // may still be read by the slower warp of the pair
    const int ep = nblk & 1;
    pair[(ep * 2 + half) * 128 + h] = make_float2(l, 0.f);
    const bool failed = bar_red_or(pair_bar, 64, !good);  // also publishes this half's sum
    if (!failed) {
      l += pair[(ep * 2 + (half ^ 1)) * 128 + h].x;
      tc_fence_after();
      // O / l (or the raw partial) of this warp's 32 heads x 128 value dims,
      // 32 dims at a time: TMEM -> registers (a row per lane) -> a swizzled
      // 32 x 32 tile in shared memory -> rows back out, four rows of 128
      // bytes per warp store instead of 32 scattered 16-byte pieces.  The
      // tiles use the first row stage: every MMA that read it completed
      // before the last PV, which this warp has seen complete.
      float* tile = reinterpret_cast<float*>(smem + OFF_KV) + sw * 1024;
      const float m_nat = m_ref * kLn2;
      const bool partial = a.splits > 1;
      const float inv = partial ? 1.f : (l > 0.f ? 1.f / l : 0.f);
      const int rsub = lane >> 3, k4 = lane & 7;  // read-back: row 4i + rsub, dims 4 k4 .. 4 k4 + 3
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t o[32];
        tmem_ld32(t_lane + 128 * half + 32 * c, o);
        tmem_ld_wait();
        __syncwarp();  // the previous chunk's tile has been read back
#pragma unroll
        for (int k = 0; k < 8; ++k)  // 16-byte piece k of row `lane`, XOR-swizzled by the row
          *reinterpret_cast<float4*>(tile + lane * 32 + ((k ^ (lane & 7)) << 2)) =
              make_float4(__uint_as_float(o[4 * k]) * inv, __uint_as_float(o[4 * k + 1]) * inv,
                          __uint_as_float(o[4 * k + 2]) * inv, __uint_as_float(o[4 * k + 3]) * inv);
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const int r = 4 * i + rsub;  // head qw*32 + r
          const float4 v4 = *reinterpret_cast<const float4*>(tile + r * 32 + ((k4 ^ (r & 7)) << 2));
          const int hr = qw * 32 + r;
          if (hr >= a.H) continue;
          const int dim = 256 * rank + 128 * half + 32 * c + 4 * k4;
          if (partial) {
            const int64_t prow = ((int64_t)t * a.splits + sp) * a.H + hr;
            *reinterpret_cast<float4*>(a.part_o + prow * kDV + dim) = v4;
          } else if (a.out_f32) {
            *reinterpret_cast<float4*>(reinterpret_cast<float*>(a.out) + ((int64_t)t * a.H + hr) * kDV + dim) = v4;
          } else {
            const __nv_bfloat162 p0 = __floats2bfloat162_rn(v4.x, v4.y), p1 = __floats2bfloat162_rn(v4.z, v4.w);
            *reinterpret_cast<uint2*>(reinterpret_cast<__nv_bfloat16*>(a.out) + ((int64_t)t * a.H + hr) * kDV + dim) =
                make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
          }
        }
      }
      if (h < a.H && rank == 0 && half == 0) {
        if (partial)
          a.part_ml[((int64_t)t * a.splits + sp) * a.H + h] = make_float2(m_nat, l);
        else if (a.lse)
          a.lse[(int64_t)t * a.H + h] = m_nat + logf(l);
      }
    } else {
      *abort_flag = 1;
    }
    __syncwarp();
  }
  if (threadIdx.x == 0 && nblk == 0) mbar_wait(q_full, 0, a.err);  // no copy in flight at exit
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // no peer still writes into this CTA's shared memory
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem, 512);
  }
}

// Merge the split partials of one (token, head): rescale to the common max.
// The (max, sum) pairs go through shared memory; the partial rows are loaded
// in batches of 8 slices, each batch's loads issued together, the first batch
// alongside the pairs (one round trip for up to 8 slices).
constexpr int kMaxSplits = 32;  // ceil(K / 64) for K <= 2048
constexpr int kCombineBatch = 8;

__global__ void __launch_bounds__(128)
k_combine(int H, int splits, const float* __restrict__ part_o, const float2* __restrict__ part_ml,
          const int32_t* __restrict__ tok_pos, void* __restrict__ out, bool out_f32, float* __restrict__ lse) {
  __shared__ float2 s_ml[kMaxSplits];
  __shared__ int s_pos;
  const int t = blockIdx.x, h = blockIdx.y, tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  const int64_t row0 = (int64_t)t * splits * H + h;  // slice i: row0 + i * H
  if (tid < splits) s_ml[tid] = __ldcg(part_ml + row0 + (int64_t)tid * H);
  if (tid == 0) s_pos = tok_pos[t];
  float4 v[kCombineBatch];
#pragma unroll
  for (int i = 0; i < kCombineBatch; ++i)
    if (i < splits) v[i] = __ldcg(reinterpret_cast<const float4*>(part_o + (row0 + (int64_t)i * H) * kDV) + tid);
  __syncthreads();
  if (s_pos < 0) return;
  float M = -INFINITY;
  for (int i = 0; i < splits; ++i)
    if (s_ml[i].y != 0.f) M = fmaxf(M, s_ml[i].x);
  float L = 0.f, o[4] = {0.f, 0.f, 0.f, 0.f};
  for (int b0 = 0; b0 < splits; b0 += kCombineBatch) {
    if (b0 > 0) {
#pragma unroll
      for (int i = 0; i < kCombineBatch; ++i)
        if (b0 + i < splits)
          v[i] = __ldcg(reinterpret_cast<const float4*>(part_o + (row0 + (int64_t)(b0 + i) * H) * kDV) + tid);
    }
#pragma unroll
    for (int i = 0; i < kCombineBatch; ++i) {
      const int k = b0 + i;
      if (k < splits && s_ml[k].y != 0.f) {  // an empty slice wrote nothing usable
        const float f = __expf(s_ml[k].x - M);
        L += s_ml[k].y * f;
        o[0] += v[i].x * f;
        o[1] += v[i].y * f;
        o[2] += v[i].z * f;
        o[3] += v[i].w * f;
      }
    }
  }
  const float inv = L > 0.f ? 1.f / L : 0.f;
  const int64_t base = ((int64_t)t * H + h) * kDV + tid * 4;
#pragma unroll
  for (int i = 0; i < 4; ++i) store_out(out, out_f32, base + i, o[i] * inv);
  if (lse && tid == 0) lse[(int64_t)t * H + h] = M + logf(L);
}

int attn_splits(int T, int K) {
  const int clusters = 74;  // 148 SMs / 2
  if (T >= clusters) return 1;
  const int want = clusters / T;
  const int most = (K + kBK - 1) / kBK;
  return want < 1 ? 1 : (want < most ? want : most);
}

int keys_per_split(int K, int splits) {
  const int ks = (K + splits - 1) / splits;
  return (ks + kBK - 1) / kBK * kBK;
}

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

// bf16 [rows, 576] map with a box of box_x x box_y and the given swizzle.
bool make_map_576(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_x, uint32_t box_y,
                  CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDQK, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  const cuuint32_t box[2] = {box_x, box_y};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t sparse_mla_partials_bytes(int T, int K, int H) {
  const int splits = attn_splits(T, K);
  if (splits == 1) return 0;
  return (size_t)T * splits * H * (kDV * sizeof(float) + sizeof(float2));
}

cudaError_t launch_sparse_mla(const SeqsDev& s, TokenMap tm, bool tm_early, const __nv_bfloat16* q,
                              const __nv_bfloat16* kv, const int32_t* idx, int K, int H, float scale, void* out,
                              bool out_f32, float* lse, void* partials, uint32_t* err, cudaStream_t st) {
  const int T = s.num_tokens;
  int splits = attn_splits(T, K);
  const int ks = keys_per_split(K, splits);
  splits = (K + ks - 1) / ks;
  float* part_o = reinterpret_cast<float*>(partials);
  float2* part_ml = reinterpret_cast<float2*>(part_o + (size_t)T * splits * H * kDV);
  CUtensorMap tq_lat, tq_rope;
  if (!make_map_576(&tq_lat, q, (uint64_t)T * H, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B) ||
      !make_map_576(&tq_rope, q, (uint64_t)T * H, 32, 128, CU_TENSOR_MAP_SWIZZLE_64B))
    return cudaErrorInvalidValue;
  static thread_local int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(k_sparse_mla_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  AttnArgs a{s, tm, kv, idx, K, H, ks, splits, tm_early, scale * kLog2e, out, out_f32, lse, part_o, part_ml, err};
  cudaError_t e = launch_pdl("sparse_mla", k_sparse_mla_tc, dim3(2 * T * splits), dim3(kThreads), (size_t)SMEM_BYTES, st, tq_lat, tq_rope,
                             a);
  if (e == cudaSuccess) e = counted(cudaGetLastError());
  if (e != cudaSuccess || splits == 1) return e;
  e = launch_pdl("sparse_mla_combine", k_combine, dim3(T, H), dim3(128), 0, st, H, splits, (const float*)part_o, (const float2*)part_ml,
                 tm.pos, out, out_f32, lse);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace dsa
