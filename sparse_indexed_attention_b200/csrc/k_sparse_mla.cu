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
// One CTA takes 64 heads of one token and one slice of its index list, and
// works on whole 576-dim rows, so no logit ever leaves the CTA.  An M = 64
// MMA keeps its rows in 16 of the 32 lanes of each TMEM lane quarter, so
// tensor memory holds, side by side:
//   lanes 0-15 of each quarter:  Q (64 heads x 576 bf16, 288 columns) -- the
//                                A operand of S = Q K^T, read from TMEM --
//                                and S as three partial sums (64 columns
//                                each: K dims split by 64-dim atom, atom a
//                                into partial a % 3);
//   lanes 16-31:                 O (64 heads x 512 fp32, all 512 columns).
// The three partials are independent accumulation chains that the tensor
// core overlaps: one chain of 36 small MMAs into a single S is bound by the
// latency of each MMA, not by its arithmetic.
//   * four loader warps resolve every selected row of the slice up front
//     (index list -> page table -> pool row, all loads independent) and copy
//     the rows block by block (64 rows, two stages) with 16-byte cp.async
//     straight into the 128-byte-swizzled operand layout: nine 8 KB atoms of
//     64 dims each;
//   * one thread issues S = Q K^T (M = 64 heads, N = 64 rows, K = 576) and
//     O += P V (M = 64, N = 256, twice, K = 64 rows) -- V is the same gathered
//     bytes read as an MN-major operand;
//   * four softmax warps, one per lane quarter: thread i and i + 16 share a
//     head and take 32 of the block's 64 logits each (online softmax, base-2
//     exponent; the running maximum only moves -- and O is rescaled in TMEM --
//     when it grows by more than 2^8, exact because O and l share it).  P goes
//     to shared memory as two bf16 terms, P = P_hi + P_lo (within 2^-16 of the
//     fp32 value), and PV runs once per term: one bf16 term alone misses the
//     accuracy bound on rows that a few selected keys dominate (relative
//     error up to 2^-8 of the spread of V, measured on the 1024-token prefill).
//   * the query tile arrives by TMA in the second row stage and the softmax
//     warps move it into TMEM before that stage's first rows; the output rows
//     leave through shared memory with one bulk copy per head row.
// Decode batches split the index list over several CTAs per (token, head
// group); k_combine merges their partials (log-sum-exp weights).
//
// FP8 latent KV cache ([P2] section 5 table, "Main attention KV cache": FP8,
// per token-head tile of 128): rows of 576 E4M3 codes with one power-of-two
// scale per 128-element tile (the last tile, the rope dims, of 64).  The
// loaders then read each row's codes (8 bytes per piece, all of a block's
// loads issued before any is used) and its scale bytes, convert to bf16 --
// exactly: an E4M3 value times a power of two has at most 4 significant bits --
// and store the same 16-byte pieces the bf16 gather would have copied; the
// MMAs, softmax and epilogue are the bf16 path's.
#include <cudaTypedefs.h>
#include <cuda_fp16.h>
#include <cuda_fp8.h>

#include "sm100.cuh"

namespace dsa {

namespace {

using namespace sm100;

constexpr int kHG = 64;                       // heads per CTA (one M = 64 tile)
constexpr int kNAtoms = kDQK / 64;            // 9: eight latent atoms + the rope atom
constexpr int kQAtom = kHG * 128;             // query atom: 64 heads x 64 dims
constexpr int kQBytes = kNAtoms * kQAtom;     // 73728
constexpr int kSParts = 3;                    // partial sums of S
constexpr int kSCols = 64;                    // TMEM columns per partial (and P row width in keys)
constexpr int kPTerm = kHG * kSCols * 2;      // one bf16 term of P: 64 heads x 64 keys, 128-byte swizzle
constexpr int kLoaders = 128;                 // warps 4-7
constexpr int kLoaderBarrier = 1;             // named barrier of the loader warps
constexpr int kNBars = 15;
constexpr int kThreads = 288;  // warps 0-3 softmax + epilogue, 4-7 load, 8 issues MMAs and owns TMEM
constexpr int kMmaWarp = 8;
constexpr int kOutRowF32 = kDV * 4 + 16;      // epilogue staging row (padded: no bank conflicts)
constexpr int kOutRowBf16 = kDV * 2 + 16;

// Block shape: BK selected rows per block (a multiple of 16, at most 64),
// NS row stages.  The library uses (64, 2): measured on all five workloads
// it beat (48, 3), whose deeper gather pipeline did not repay the larger
// number of (issue-bound) QK MMAs per selected row.
template <int BK_, int NS_>
struct AttnCfg {
  static constexpr int BK = BK_, NS = NS_;
  static constexpr int ATOM = BK * 128;                    // BK rows x 64 bf16 dims, 128-byte swizzle
  static constexpr int STAGE = kNAtoms * ATOM;
  static constexpr int MAX_BLOCKS = (kMaxK + BK - 1) / BK;
  static constexpr int OFF_KV = 0;                         // stage 0 stages the index lists at first
  static constexpr int OFF_Q = (NS - 1) * STAGE;           // the query tile lands in the last stage (and on)
  static constexpr int OFF_P = NS * STAGE;                 // [2 buffers][hi, lo]
  static constexpr int OFF_ROWS = OFF_P + 2 * 2 * kPTerm;  // [block][BK] pool rows of the slice (-1 = masked)
  static constexpr int OFF_MASK = OFF_ROWS + MAX_BLOCKS * BK * 4;  // [block] 64-bit validity masks
  static constexpr int OFF_BAR = OFF_MASK + MAX_BLOCKS * 8;
  static constexpr int OFF_MISC = OFF_BAR + kNBars * 8;
  static constexpr int SMEM = OFF_MISC + 16 + 1024;        // slack for 1024-byte alignment
  static constexpr uint32_t IDESC_QK = make_idesc_major(true, kHG, BK, 0, 0);  // S = Q K^T, both K-major
  static_assert(BK % 16 == 0 && BK <= kSCols, "block shape");
  static_assert(SMEM <= 227 * 1024, "shared memory");
  static_assert(ATOM % 1024 == 0 && OFF_Q % 1024 == 0 && OFF_P % 1024 == 0, "swizzle atoms need 1024-B alignment");
  static_assert(OFF_Q + kQBytes <= OFF_ROWS, "the query tile fits in the last stage and the P buffers");
  static_assert(kHG * kOutRowF32 <= NS * STAGE, "epilogue staging fits in the row stages");
  static_assert(2 * kMaxK * 4 <= STAGE, "index staging fits in stage 0");
};
using Cfg = AttnCfg<64, 2>;

// TMEM map: lane offset << 16 | column
constexpr uint32_t kTmemS = 288;             // S partials at columns 288, 352, 416 of lanes 0-15 (Q at 0)
constexpr uint32_t kTmemO = 16u << 16;       // O: lanes 16-31, columns 0-511

constexpr uint32_t IDESC_PV = make_idesc_major(true, kHG, 256, 0, 1);  // O += P V, V MN-major
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
constexpr float kRescaleThreshold = 8.0f;     // log2 units

// 2^x from the MUFU unit (approximate, subnormal results flushed to 0;
// ex2(-inf) = +0).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// 8 bytes from global memory through the read-only path.
__device__ __forceinline__ uint2 ld_nc_v2(const void* p) {
  uint2 v;
  asm volatile("ld.global.nc.v2.u32 {%0, %1}, [%2];" : "=r"(v.x), "=r"(v.y) : "l"(p));
  return v;
}

// 2^(byte - 127) for a tile-scale byte, exact (2^-127 is the subnormal 0x00400000).
__device__ __forceinline__ float tile_scale(uint32_t byte) {
  return byte == 0u ? __uint_as_float(0x00400000u) : __uint_as_float(byte << 23);
}

// Eight E4M3 codes (little-endian: element k in byte k) times a power-of-two
// scale, as eight bf16 (element 2i in the low half of word i).  Exact: an
// E4M3 value is an fp16 value, and times 2^e it has at most 4 significant bits.
__device__ __forceinline__ uint4 e4m3x8_to_bf16x8(uint2 codes, float sc) {
  uint32_t o[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t w = i < 2 ? codes.x : codes.y;
    const __nv_fp8x2_storage_t pair = (__nv_fp8x2_storage_t)((w >> (16 * (i & 1))) & 0xFFFFu);
    const __half2_raw hr = __nv_cvt_fp8x2_to_halfraw2(pair, __NV_E4M3);
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&hr));
    const __nv_bfloat162 b = __floats2bfloat162_rn(f.x * sc, f.y * sc);
    o[i] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(o[0], o[1], o[2], o[3]);
}

__device__ __forceinline__ void store_out(void* out, bool f32, int64_t i, float v) {
  if (f32)
    reinterpret_cast<float*>(out)[i] = v;
  else
    reinterpret_cast<__nv_bfloat16*>(out)[i] = __float2bfloat16(v);
}

__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
  return smem_desc(saddr, lbo, sbo, 2);
}

// A descriptor moved by `bytes` (a compile-time offset inside the operand):
// the start address sits in the low 14 bits as address / 16 and stays below
// 2^14 for any shared-memory address, so the move is one add.  The issuing
// thread builds each operand's base descriptor once per block.
__device__ __forceinline__ uint64_t desc_at(uint64_t base, uint32_t bytes) { return base + (bytes >> 4); }

struct AttnArgs {
  SeqsDev s;
  TokenMap tm;
  const __nv_bfloat16* kv;  // latent pool [rows, 576]
  const uint8_t* kv8;       // FP8 cache: E4M3 codes [rows, 576] (kv unused)
  const uint8_t* kv8_scale; // FP8 cache: per row 8 bytes, byte j = exponent + 127 of tile j (0..4)
  const int32_t* idx;
  int K, H, G, ks, splits;  // G head groups of 64; ks selected slots per split
  bool tm_early;            // the token map was written two or more launches back
  float scale_log2;         // scale * log2(e)
  void* out;
  bool out_f32;
  float* lse;
  float* part_o;
  float2* part_ml;
  uint32_t* err;
  uint64_t wait_ns;         // limit of each wait for another role's progress
};

// The query tile (64 heads x 576 dims, 128-byte-swizzled atoms in shared
// memory) into TMEM as the A operand of S = Q K^T: warp q writes heads
// 16q .. 16q+15, thread i (i < 16) dims [0, 288) and thread i + 16 dims
// [288, 576) of head 16q + i, as bf16 pairs (column c = dims 2c, 2c + 1).
// Heads at or past H are zero.
__device__ __forceinline__ void query_to_tmem(const uint8_t* qs, bool valid, int hr, int half, uint32_t t_q) {
#pragma unroll
  for (int chunk = 0; chunk < 9; ++chunk) {  // 32 dims = 4 pieces of 16 bytes = 16 TMEM columns
    uint32_t r[16];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int d = 288 * half + 32 * chunk + 8 * k;  // first dim of the piece
      const int at = d >> 6, piece = (d & 63) >> 3;
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (valid) v = *reinterpret_cast<const uint4*>(qs + at * kQAtom + hr * 128 + ((piece ^ (hr & 7)) << 4));
      r[4 * k] = v.x;
      r[4 * k + 1] = v.y;
      r[4 * k + 2] = v.z;
      r[4 * k + 3] = v.w;
    }
    tmem_st16x2_16<144>(t_q + 16 * chunk, r);
  }
}

template <int BK, int NS, bool kKv8>
__global__ void __launch_bounds__(kThreads, 1)
k_sparse_mla_tc(const __grid_constant__ CUtensorMap tq, const AttnArgs a) {
  using C = AttnCfg<BK, NS>;
  constexpr int OFF_KV = C::OFF_KV, OFF_P = C::OFF_P;
  constexpr int kAtom = C::ATOM, kStageBytes = C::STAGE, kStages = NS, kBK = BK;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024 - (smem_u32(smem_raw) & 1023)) & 1023);
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_tma = bars + 0;      // the query tile has landed in stage 1
  uint64_t* q_full = bars + 1;     // the query is in TMEM and stage 1 is free (one arrival per softmax warp)
  uint64_t* kv_full = bars + 2;    // [NS] rows of block j (stage j % NS) landed
  uint64_t* kv_empty = bars + 5;   // [NS] PV of the stage's block completed
  uint64_t* s_full = bars + 8;     // S of block j in TMEM
  uint64_t* s_empty = bars + 9;    // S read by every softmax warp
  uint64_t* p_full = bars + 10;    // [2] P of block j (buffer j & 1) in shared memory
  uint64_t* o_done = bars + 12;    // [2] PV of block i (parity by i & 1) has completed
  uint64_t* mma_drain = bars + 14; // every MMA this CTA issued has completed
  int32_t* ring_rows = reinterpret_cast<int32_t*>(smem + C::OFF_ROWS);
  uint64_t* ring_mask = reinterpret_cast<uint64_t*>(smem + C::OFF_MASK);
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + C::OFF_MISC);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + C::OFF_MISC + 4);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int cta = blockIdx.x;
  const int g = cta % a.G, rest = cta / a.G;  // the head groups of a (token, slice) are neighbours (shared rows in L2)
  const int sp = rest % a.splits, t = rest / a.splits;
  const int kbeg = sp * a.ks;
  const int kend = min(a.K, kbeg + a.ks);

  if (threadIdx.x == 0) {
    mbar_init(q_tma, 1);
    mbar_init(q_full, 4);
    for (int i = 0; i < kStages; ++i) {
      mbar_init(&kv_full[i], kLoaders + 1);  // every loader's copies + the mask's publisher
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(s_full, 1);
    mbar_init(s_empty, 4);
    for (int i = 0; i < 2; ++i) {
      mbar_init(&p_full[i], 4);  // one arrival per softmax warp
      mbar_init(&o_done[i], 1);
    }
    mbar_init(mma_drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kMmaWarp) {
    tmem_alloc(tmem_slot, 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;
  if (threadIdx.x == 0) {  // q is an input of the call: its load overlaps the wait below
    prefetch_tmap(&tq);
    mbar_arrive_expect_tx(q_tma, kQBytes);
    for (int at = 0; at < kNAtoms; ++at)
      tma_load_2d(smem + C::OFF_Q + at * kQAtom, &tq, q_tma, 64 * at, t * a.H + kHG * g);
  }
  // the token map can be read before the wait when it does not come from
  // the kernel just before; the index lists always do
  int pos = a.tm_early ? a.tm.pos[t] : 0, b = a.tm_early ? a.tm.seq[t] : 0;
  if (a.tm_early && warp == 4 && pos >= 0) {
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

  if (warp >= 4 && warp < kMmaWarp && nblk > 0) {
    // ---------------------------------------------------------------- loaders
    const int li = threadIdx.x - 128;  // 0 .. 127
    const int lw = warp - 4;           // loader warp 0 .. 3
    // Pool rows of every block of the slice, resolved up front in three
    // passes whose loads are all independent: the index list, then the page
    // ids (both staged by cp.async in stage 0, which block 0's copies fill
    // only after the last pass), then rows and masks (row -1 = masked).
    {
      const int nkeys = kend - kbeg;
      int32_t* s_sidx = reinterpret_cast<int32_t*>(smem + OFF_KV);
      int32_t* s_page = s_sidx + kMaxK;
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
      for (int w32 = lw; w32 < 2 * nblk; w32 += 4) {  // 32 rows per warp -> half a block's mask
        const int r = 32 * (w32 & 1) + lane;         // row of block w32 / 2 (rows >= BK never count)
        const uint32_t m = __ballot_sync(0xffffffffu, r < kBK && ring_rows[(w32 >> 1) * kBK + r] >= 0);
        if (lane == 0) reinterpret_cast<uint32_t*>(ring_mask)[w32] = m;
      }
    }
    const uint32_t kv_smem = smem_u32(smem + OFF_KV);
    const char* kv_base = reinterpret_cast<const char*>(a.kv);
    const int rsub = lane >> 3, piece = lane & 7;  // a warp copies 4 rows x 128 bytes of one atom at a time
    constexpr int kQuads = BK / 4;  // row quads per block
    bool failed = bar_red_or(kLoaderBarrier, kLoaders, false);
    // FP8 cache: this thread's pieces of a block (4 rows x 9 atoms of 8 codes)
    // and its rows' scale words, loaded one block ahead: the next block's loads
    // are issued as soon as this block's pieces are stored, so their latency
    // overlaps the wait for the next free stage
    static_assert(!kKv8 || BK / 4 == 16, "four row quads per loader warp");
    uint2 raw[4][kNAtoms], scl[4];
    auto load_block = [&](int jb) {
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int r = 4 * (lw + 4 * u) + rsub;
        const int row = ring_rows[jb * kBK + r];
        if (row >= 0) {
          const uint8_t* src = a.kv8 + (int64_t)row * kDQK + 8 * piece;
#pragma unroll
          for (int at = 0; at < kNAtoms; ++at) raw[u][at] = ld_nc_v2(src + 64 * at);
          scl[u] = ld_nc_v2(a.kv8_scale + (int64_t)row * 8);
        } else {  // masked row: zeros, as the bf16 gather's zero fill
#pragma unroll
          for (int at = 0; at < kNAtoms; ++at) raw[u][at] = make_uint2(0u, 0u);
          scl[u] = make_uint2(0x7F7F7F7Fu, 0x7Fu);
        }
      }
    };
    if constexpr (kKv8) {
      if (!failed) load_block(0);
    }
    for (int j = 0; j < nblk && !failed; ++j) {
      const int stage = j % kStages;
      // the PV of the stage's previous block has completed
      bool ok = mbar_wait(&kv_empty[stage], ((j / kStages) & 1) ^ 1, a.err, a.wait_ns);
      // the last stage first holds the query tile
      if (j == NS - 1) ok = ok && mbar_wait(q_full, 0, a.err, a.wait_ns);
      if (ok && kKv8) {
        // FP8 cache: convert the block loaded ahead and store its pieces
        uint8_t* dst0 = smem + OFF_KV + stage * kStageBytes;
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int r = 4 * (lw + 4 * u) + rsub;
          uint8_t* drow = dst0 + r * 128 + ((((uint32_t)piece) ^ ((uint32_t)r & 7u)) << 4);
#pragma unroll
          for (int at = 0; at < kNAtoms; ++at) {
            const int tile = at >> 1;  // atom at holds dims 64 at .. 64 at + 63
            const uint32_t byte = (tile < 4 ? (scl[u].x >> (8 * tile)) : scl[u].y) & 0xFFu;
            *reinterpret_cast<uint4*>(drow + at * kAtom) = e4m3x8_to_bf16x8(raw[u][at], tile_scale(byte));
          }
        }
        fence_proxy_async_smem();  // the MMAs read these stores through the async proxy
        if (j + 1 < nblk) load_block(j + 1);
      } else if (ok) {
        // one row per (warp, quad): its pool row is looked up once, then the
        // nine 128-byte pieces (one per atom) go out back to back; a warp's
        // 32 copies of one atom fill 512 contiguous bytes (no bank conflict)
        const uint32_t dst0 = kv_smem + stage * kStageBytes;
#pragma unroll 1
        for (int qd = lw; qd < kQuads; qd += 4) {
          const int r = 4 * qd + rsub;
          const int row = ring_rows[j * kBK + r];
          const bool v = row >= 0;
          const char* src = kv_base + (v ? (int64_t)row * (kDQK * 2) : 0) + 16 * piece;
          const uint32_t dst = dst0 + r * 128 + ((((uint32_t)piece) ^ ((uint32_t)r & 7u)) << 4);
#pragma unroll
          for (int at = 0; at < kNAtoms; ++at) cp_async_16_zfill(dst + at * kAtom, src + 128 * at, v ? 16u : 0u);
        }
      }
      if constexpr (kKv8)
        mbar_arrive(&kv_full[stage]);            // the stores above are done
      else
        cp_async_mbar_arrive(&kv_full[stage]);   // counts once this thread's copies land
      if (li == 0) mbar_arrive(&kv_full[stage]);  // releases the masks read by the softmax warps
      failed = bar_red_or(kLoaderBarrier, kLoaders, !ok || *abort_flag != 0);
      if (failed) *abort_flag = 1;
    }
    cp_async_wait_all();  // nothing this thread copies is still in flight at exit
    __syncwarp();
  } else if (warp == kMmaWarp && nblk > 0) {
    // ---------------------------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint32_t kv_base = smem_u32(smem + OFF_KV);
      const uint32_t p_base = smem_u32(smem + OFF_P);
      bool ok = mbar_wait(q_full, 0, a.err, a.wait_ns);
      tc_fence_after();
      // Issue whichever is ready, PV first (it frees a row stage):
      //   PV(i) once P(i) is in shared memory;
      //   QK(j) once block j's rows have landed and S(j-1) has been read.
      int nq = 0, np = 0;  // next block to score / to accumulate
      uint64_t idle_since = 0;
      while (ok && np < nblk) {
        if (*abort_flag) {
          ok = false;
          break;
        }
        if (np < nq && mbar_test_wait(&p_full[np & 1], (np >> 1) & 1)) {
          fence_proxy_async_smem();  // P was written by the softmax threads (generic proxy)
          tc_fence_after();
          const uint64_t vd = sw128_desc(kv_base + (np % kStages) * kStageBytes, kAtom, 1024);
          const uint64_t pd = sw128_desc(p_base + (np & 1) * 2 * kPTerm, 16, 1024);
          const bool acc0 = np > 0;
#pragma unroll
          for (int term = 0; term < 2; ++term)
#pragma unroll
            for (int kk = 0; kk < kBK / 16; ++kk)
#pragma unroll
              for (int half = 0; half < 2; ++half)  // the halves alternate: independent chains
                mma_ss<true>(tmem + kTmemO + 256 * half, desc_at(pd, term * kPTerm + kk * 32),
                             desc_at(vd, 4 * half * kAtom + kk * 2048), IDESC_PV, acc0 || term > 0 || kk > 0);
          mma_commit(&kv_empty[np % kStages]);
          mma_commit(&o_done[np & 1]);
          ++np;
          idle_since = 0;
        } else if (nq < nblk && nq < np + 2 && mbar_test_wait(&kv_full[nq % kStages], (nq / kStages) & 1) &&
                   (nq == 0 || mbar_test_wait(s_empty, (nq - 1) & 1))) {
          fence_proxy_async_smem();  // the rows were written by cp.async (generic proxy)
          tc_fence_after();
          const uint64_t kd = sw128_desc(kv_base + (nq % kStages) * kStageBytes, 16, 1024);
          // atom at -> partial at % 3; consecutive MMAs go to different partials
#pragma unroll
          for (int grp = 0; grp < kNAtoms / kSParts; ++grp)
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)  // K step of 16 dims = 8 TMEM columns of Q
#pragma unroll
              for (int part = 0; part < kSParts; ++part) {
                const int at = kSParts * grp + part;
                mma_ts_bf16(tmem + kTmemS + kSCols * part, tmem + 32 * at + 8 * kk,
                            desc_at(kd, at * kAtom + kk * 32), C::IDESC_QK, (grp | kk) != 0);
              }
          mma_commit(s_full);
          ++nq;
          idle_since = 0;
        } else {
          const uint64_t now = globaltimer();
          if (idle_since == 0) {
            idle_since = now;
          } else if (now - idle_since > a.wait_ns) {
            raise_error(a.err, kErrTimeout);
            ok = false;
          }
          __nanosleep(32);
        }
      }
      if (!ok) *abort_flag = 1;
      // drain, also after a failed wait: no MMA still reads shared memory or
      // writes TMEM when the CTA deallocates and exits
      mma_commit(mma_drain);
      mbar_wait(mma_drain, 0, a.err, kDrainLimitNs);
    }
    __syncwarp();
  } else if (warp < 4) {
    // ---------------------------------------------------------------- softmax / epilogue
    // Warp q reads lane quarter q: Q and S rows at lanes 0-15, O rows at
    // lanes 16-31, head hr = 16q + (lane & 15).  Lanes i and i + 16 share the
    // head: kh = 0 / 1 takes logits [0, 32) / [32, 64) of every block and
    // value dims [0, 256) / [256, 512) of O.
    const int q = warp;
    const int hr = 16 * q + (lane & 15);
    const int kh = lane >> 4;
    const int head = kHG * g + hr;
    const bool mine = head < a.H;
    const uint32_t t_s = tmem + ((uint32_t)(32 * q) << 16) + kTmemS;
    const uint32_t t_o = tmem + ((uint32_t)(32 * q) << 16) + kTmemO;
    bool good = true;
    if (nblk > 0) {
      good = __all_sync(0xffffffffu, mbar_wait(q_tma, 0, a.err, a.wait_ns));
      if (good) {
        query_to_tmem(smem + C::OFF_Q, mine, hr, kh, tmem + ((uint32_t)(32 * q) << 16));
        tmem_st_wait();
      }
      tc_fence_before();
      __syncwarp();
      if (good && lane == 0) mbar_arrive(q_full);
    }
    const float sc = a.scale_log2;
    float m_ref = -INFINITY, l = 0.f;  // l: this thread's share of the head's sum
    for (int j = 0; j < nblk && good; ++j) {
      const int sb = j & 1;
      const int stage = j % kStages;
      good = __all_sync(0xffffffffu, !*abort_flag && mbar_wait(s_full, j & 1, a.err, a.wait_ns));
      if (!good) break;
      uint32_t v[32], w[32];
      float s[32];
      tc_fence_after();
      tmem_ld16x2_32<32>(t_s, v);
      tmem_ld16x2_32<32>(t_s + kSCols, w);
      tmem_ld_wait_regs(v);
      tmem_ld_wait_regs(w);
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] = __uint_as_float(v[i]) + __uint_as_float(w[i]);
      tmem_ld16x2_32<32>(t_s + 2 * kSCols, v);
      tmem_ld_wait_regs(v);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(s_empty);
      // validity of the block's rows (published before the stage completed)
      good = __all_sync(0xffffffffu, mbar_wait(&kv_full[stage], (j / kStages) & 1, a.err, a.wait_ns));
      if (!good) break;
      const uint32_t m32 = (uint32_t)(ring_mask[j] >> (32 * kh));
#pragma unroll
      for (int i = 0; i < 32; ++i) s[i] += __uint_as_float(v[i]);
      if (m32 != 0xffffffffu) {  // masked rows (padding, bad indices) never count
#pragma unroll
        for (int i = 0; i < 32; ++i) s[i] = ((m32 >> i) & 1u) ? s[i] : -INFINITY;
      }
      // maxima as trees (depth 5), not chains
      float mx[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) mx[i] = fmaxf(s[i], s[i + 16]);
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) mx[i] = fmaxf(mx[i], mx[i + w]);
      float mraw = fmaxf(mx[0], __shfl_xor_sync(0xffffffffu, mx[0], 16));
      float mblk;
      if (sc > 0.f) {
        mblk = mraw == -INFINITY ? -INFINITY : mraw * sc;
      } else {
        // scale <= 0 (allowed, if odd): the largest scaled logit comes from
        // the smallest unmasked raw one
        float mneg = INFINITY;
#pragma unroll
        for (int i = 0; i < 32; ++i) mneg = fminf(mneg, s[i] == -INFINITY ? INFINITY : s[i]);
        mneg = fminf(mneg, __shfl_xor_sync(0xffffffffu, mneg, 16));
        mblk = mraw == -INFINITY ? -INFINITY : mneg * sc;
      }
      const bool move = mblk > m_ref + kRescaleThreshold;
      const float m_new = move ? mblk : m_ref;
      const float alpha = move ? exp2f(m_ref - m_new) : 1.f;  // exp2(-inf) = 0 on the first block
      const float mu = m_new == -INFINITY ? 0.f : m_new;      // nothing unmasked yet: every term is 0
      uint32_t pk[16], pl[16];
      float ps[16];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        // masked: s = -inf and sc > 0 give ex2(-inf) = 0; sc <= 0 takes the select
        const float x0 = fmaf(s[2 * i], sc, -mu), x1 = fmaf(s[2 * i + 1], sc, -mu);
        const float e0 = sc > 0.f ? ex2_ftz(x0) : (s[2 * i] == -INFINITY ? 0.f : ex2_ftz(x0));
        const float e1 = sc > 0.f ? ex2_ftz(x1) : (s[2 * i + 1] == -INFINITY ? 0.f : ex2_ftz(x1));
        ps[i] = e0 + e1;
        const __nv_bfloat162 hi = __floats2bfloat162_rn(e0, e1);
        const uint32_t hb = *reinterpret_cast<const uint32_t*>(&hi);
        const __nv_bfloat162 lo =
            __floats2bfloat162_rn(e0 - __uint_as_float(hb << 16), e1 - __uint_as_float(hb & 0xFFFF0000u));
        pk[i] = hb;
        pl[i] = *reinterpret_cast<const uint32_t*>(&lo);
      }
#pragma unroll
      for (int w = 8; w > 0; w >>= 1)
#pragma unroll
        for (int i = 0; i < w; ++i) ps[i] += ps[i + w];
      const float psum = ps[0];
      // P(j) into buffer j & 1 once PV(j-2), its last reader, has completed
      // (with two stages QK(j) could not start before that): row hr, this
      // thread's four 16-byte pieces of keys [32 kh, 32 kh + 32), each term in
      // its own 128-byte-swizzled tile
      if (NS > 2 && j >= 2) {
        good = __all_sync(0xffffffffu, mbar_wait(&o_done[j & 1], ((j - 2) >> 1) & 1, a.err, a.wait_ns));
        if (!good) break;
      }
      uint8_t* prow = smem + OFF_P + sb * 2 * kPTerm + hr * 128;
#pragma unroll
      for (int c = 0; c < 4; ++c) {
        const uint32_t off = (((uint32_t)(4 * kh + c)) ^ ((uint32_t)hr & 7u)) << 4;
        *reinterpret_cast<uint4*>(prow + off) = make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
        *reinterpret_cast<uint4*>(prow + kPTerm + off) =
            make_uint4(pl[4 * c], pl[4 * c + 1], pl[4 * c + 2], pl[4 * c + 3]);
      }
      fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
      // TMEM loads/stores are warp-wide: if any head of the warp moved its
      // maximum, the warp rescales its heads' rows of O (alpha = 1 leaves a
      // row exact), once PV(j-1) -- the last writer of O -- has completed
      if (j >= 1 && __any_sync(0xffffffffu, move && m_ref != -INFINITY)) {
        good = __all_sync(0xffffffffu, mbar_wait(&o_done[(j - 1) & 1], ((j - 1) >> 1) & 1, a.err, a.wait_ns));
        if (!good) break;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld16x2_32<256>(t_o + 32 * c, o);
          tmem_ld_wait_regs(o);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = __float_as_uint(__uint_as_float(o[i]) * alpha);
          tmem_st16x2_32<256>(t_o + 32 * c, o);
        }
      }
      l = l * alpha + psum;
      m_ref = m_new;
      tmem_st_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[sb]);
    }
    // epilogue: O / l for this thread's head and 256 value dims, staged in
    // the row stages (every MMA that read them has completed: o_done of the
    // last block tracks all of them) and written with one bulk copy per row
    if (nblk > 0) {
      good = good && __all_sync(0xffffffffu, mbar_wait(&o_done[(nblk - 1) & 1], ((nblk - 1) >> 1) & 1, a.err,
                                                       a.wait_ns));
      const float lt = l + __shfl_xor_sync(0xffffffffu, l, 16);
      if (good) {
        tc_fence_after();
        const bool partial = a.splits > 1;
        const bool f32 = partial || a.out_f32;
        const float inv = partial ? 1.f : (lt > 0.f ? 1.f / lt : 0.f);
        const int64_t orow = partial ? (((int64_t)t * a.splits + sp) * a.H + head) : ((int64_t)t * a.H + head);
        uint8_t* srow = smem + OFF_KV + hr * (f32 ? kOutRowF32 : kOutRowBf16);
        uint32_t on[32];
        tmem_ld16x2_32<256>(t_o, on);
#pragma unroll 1
        for (int c = 0; c < 8; ++c) {
          uint32_t o[32];
          tmem_ld_wait_regs(on);
#pragma unroll
          for (int i = 0; i < 32; ++i) o[i] = on[i];
          if (c + 1 < 8) tmem_ld16x2_32<256>(t_o + 32 * (c + 1), on);  // the next chunk's load overlaps this one's stores
          const int dim = 256 * kh + 32 * c;
          if (f32) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              *reinterpret_cast<float4*>(srow + dim * 4 + 16 * i) =
                  make_float4(__uint_as_float(o[4 * i]) * inv, __uint_as_float(o[4 * i + 1]) * inv,
                              __uint_as_float(o[4 * i + 2]) * inv, __uint_as_float(o[4 * i + 3]) * inv);
          } else {
#pragma unroll
            for (int i = 0; i < 4; ++i) {
              uint32_t w4[4];
#pragma unroll
              for (int k = 0; k < 4; ++k) {
                const __nv_bfloat162 p2 = __floats2bfloat162_rn(__uint_as_float(o[8 * i + 2 * k]) * inv,
                                                                 __uint_as_float(o[8 * i + 2 * k + 1]) * inv);
                w4[k] = *reinterpret_cast<const uint32_t*>(&p2);
              }
              *reinterpret_cast<uint4*>(srow + dim * 2 + 16 * i) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
            }
          }
        }
        fence_proxy_async_smem();  // the bulk copy reads the staged row (async proxy)
        __syncwarp();
        if (mine && kh == 0) {
          void* dst = partial ? (void*)(a.part_o + orow * kDV)
                              : (a.out_f32 ? (void*)(reinterpret_cast<float*>(a.out) + orow * kDV)
                                           : (void*)(reinterpret_cast<__nv_bfloat16*>(a.out) + orow * kDV));
          bulk_store(dst, srow, f32 ? kDV * 4 : kDV * 2);
          bulk_commit();
          const float m_nat = m_ref * kLn2;
          if (partial)
            a.part_ml[orow] = make_float2(m_nat, lt);
          else if (a.lse)
            a.lse[orow] = m_nat + logf(lt);
          bulk_wait_read();  // the staged row stays until the copy has read it
        }
      } else {
        *abort_flag = 1;
      }
    }
    __syncwarp();
  }
  // drain: the query tile's copy has landed before the CTA exits (its
  // consumers may have given up waiting, or never run when nblk == 0)
  if (threadIdx.x == 0) mbar_wait(q_tma, 0, a.err, kDrainLimitNs);
  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
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

constexpr int kSplitSms = 148;  // SMs the split decision fills (a host-only constant: no device query)

int head_groups(int H) { return (H + kHG - 1) / kHG; }

// Batches with fewer (token, head group) units than SMs split each index
// list over several CTAs (whose partials k_combine merges).
int attn_splits(int T, int K, int H) {
  const int64_t units = (int64_t)T * head_groups(H);
  if (units >= kSplitSms) return 1;
  const int want = kSplitSms / (int)units;
  int most = (K + Cfg::BK - 1) / Cfg::BK;
  if (most > kMaxSplits) most = kMaxSplits;
  return want < 1 ? 1 : (want < most ? want : most);
}

int keys_per_split(int K, int splits, int bk) {
  const int ks = (K + splits - 1) / splits;
  return (ks + bk - 1) / bk * bk;
}

template <int BK, int NS, bool kKv8>
cudaError_t launch_attn(const CUtensorMap& tq, const AttnArgs& a, int64_t ctas, cudaStream_t st) {
  using C = AttnCfg<BK, NS>;
  static thread_local int attr_dev = -1;
  int dev = 0;
  cudaGetDevice(&dev);
  if (attr_dev != dev) {
    cudaError_t e = cudaFuncSetAttribute(k_sparse_mla_tc<BK, NS, kKv8>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         C::SMEM);
    if (e != cudaSuccess) return e;
    attr_dev = dev;
  }
  return launch_pdl("sparse_mla", k_sparse_mla_tc<BK, NS, kKv8>, dim3((unsigned)ctas), dim3(kThreads),
                    (size_t)C::SMEM, st, tq, a);
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

// bf16 [rows, 576] map with a box of 64 dims x 64 rows and the 128-byte swizzle.
bool make_map_576(CUtensorMap* m, const void* base, uint64_t rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {(cuuint64_t)kDQK, rows};
  const cuuint64_t strides[1] = {(cuuint64_t)kDQK * 2};
  const cuuint32_t box[2] = {64, (cuuint32_t)kHG};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

size_t sparse_mla_partials_bytes(int T, int K, int H) {
  const int splits = attn_splits(T, K, H);
  if (splits == 1) return 0;
  return (size_t)T * splits * H * (kDV * sizeof(float) + sizeof(float2));
}

cudaError_t launch_sparse_mla(const SeqsDev& s, TokenMap tm, bool tm_early, const __nv_bfloat16* q, const void* kv,
                              const uint8_t* kv8_scale, const int32_t* idx, int K, int H, float scale, void* out,
                              bool out_f32, float* lse, void* partials, uint32_t* err, cudaStream_t st) {
  const int T = s.num_tokens;
  const int G = head_groups(H);
  int splits = attn_splits(T, K, H);
  const int ks = keys_per_split(K, splits, Cfg::BK);
  splits = (K + ks - 1) / ks;
  float* part_o = reinterpret_cast<float*>(partials);
  float2* part_ml = reinterpret_cast<float2*>(part_o + (size_t)T * splits * H * kDV);
  CUtensorMap tq;
  if (!make_map_576(&tq, q, (uint64_t)T * H)) return cudaErrorInvalidValue;
  const bool kv8 = kv8_scale != nullptr;
  AttnArgs a{s,
             tm,
             kv8 ? nullptr : static_cast<const __nv_bfloat16*>(kv),
             kv8 ? static_cast<const uint8_t*>(kv) : nullptr,
             kv8_scale,
             idx,
             K, H, G, ks, splits, tm_early, scale * kLog2e, out, out_f32, lse, part_o, part_ml, err, wait_limit_ns()};
  const int64_t ctas = (int64_t)T * G * splits;
  if (ctas > 0x7fffffff) return cudaErrorInvalidValue;
  cudaError_t e = kv8 ? launch_attn<Cfg::BK, Cfg::NS, true>(tq, a, ctas, st)
                      : launch_attn<Cfg::BK, Cfg::NS, false>(tq, a, ctas, st);
  if (e == cudaSuccess) e = counted(cudaGetLastError());
  if (e != cudaSuccess || splits == 1) return e;
  e = launch_pdl("sparse_mla_combine", k_combine, dim3(T, H), dim3(128), 0, st, H, splits, (const float*)part_o,
                 (const float2*)part_ml, tm.pos, out, out_f32, lse);
  if (e != cudaSuccess) return e;
  return counted(cudaGetLastError());
}

}  // namespace dsa
