// Internal declarations shared by the libdsa translation units (not part of
// the public ABI, which is include/dsa.h).
#pragma once
#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <utility>

#include "../../include/dsa.h"

namespace dsa {

// Fixed sizes of the path (see include/dsa.h).
constexpr int kPage = 64;        // tokens per page
constexpr int kHI = 64;          // index heads
constexpr int kDI = 128;         // index dim
constexpr int kDQK = 576;        // latent key dims (512 latent + 64 rope)
constexpr int kDV = 512;         // latent value dims
constexpr int kMaxK = 2048;

// Bits of the sticky device error word (first word of the workspace).
constexpr uint32_t kErrBadIndex = 1u;
constexpr uint32_t kErrTimeout = 2u;

__device__ __forceinline__ void raise_error(uint32_t* err, uint32_t bit) {
  if ((*(volatile uint32_t*)err & bit) == 0) atomicOr(err, bit);
}

// Order-preserving 32-bit key of a score: larger score <=> larger key;
// -0.0 ranks equal to +0.0.  Shared by Top-K and the indexer epilogue (which
// builds Top-K's first-digit histogram while it writes the scores).
__device__ __forceinline__ uint32_t order_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Top-K's first digit: the top 11 key bits.
constexpr int kTopkHistBins = 2048;
constexpr int kTopkLowBits = 21;

// Adds one to hist[bin]; lanes of the warp holding the same bin add once.
// Every lane of the warp must call it (active or not).
__device__ __forceinline__ void hist_add(uint32_t* hist, uint32_t bin, bool active) {
  const uint32_t act = __ballot_sync(0xffffffffu, active);
  if (!active) return;
  const uint32_t peers = __match_any_sync(act, bin);
  if ((__ffs(peers) - 1) == (int)(threadIdx.x & 31)) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
}

// Per query token: its sequence and absolute position (-1 = invalid token).
struct TokenMap {
  const int32_t* seq;
  const int32_t* pos;
};

// Physical pool row of logical position s of sequence b, or -1 (and the error
// bit) when the page id is outside the pool.
__device__ __forceinline__ int64_t phys_row(const int32_t* __restrict__ page_table, int max_pages,
                                            int num_phys_pages, int b, int s, uint32_t* err) {
  int page = __ldg(page_table + (int64_t)b * max_pages + (s >> 6));
  if (page < 0 || page >= num_phys_pages) {
    raise_error(err, kErrBadIndex);
    return -1;
  }
  return (int64_t)page * kPage + (s & (kPage - 1));
}

// Device-side batch geometry passed by value to kernels.
struct SeqsDev {
  int batch, num_tokens, max_pages, num_phys_pages, max_ctx;
  const int32_t* q_seq_start;
  const int32_t* ctx_len;
  const int32_t* page_table;
};

// Programmatic dependent launch: every kernel of the path is launched with
// programmatic stream serialization, so its launch and its set-up (barrier
// init, TMEM allocation, tensor-map prefetch) overlap the previous kernel's
// tail.  A kernel touches global memory only after pdl_wait(), which returns
// once the previous grid has completed and its writes are visible, and lets
// the next kernel launch (pdl_trigger) right after.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// Optional per-launch timing (dsa_launch_timing): event 0 before a call's
// first kernel, event i+1 after its kernel i.
constexpr int kMaxTimedLaunches = 16;
struct LaunchTimer {
  int device = -1;     // the events exist, on this device, when >= 0
  bool armed = false;  // the current call records events
  int n = 0;           // kernels timed in the current / last timed call
  cudaEvent_t ev[kMaxTimedLaunches + 1] = {};
  const char* name[kMaxTimedLaunches] = {};
};
extern thread_local LaunchTimer g_timer;

// Start of an entry point's launches on stream st.
__host__ inline void timer_begin(cudaStream_t st) {
  g_timer.armed = g_timer.device >= 0;
  g_timer.n = 0;
  if (g_timer.armed) cudaEventRecord(g_timer.ev[0], st);
}

__host__ inline void timer_mark(const char* name, cudaStream_t st) {
  if (!g_timer.armed || g_timer.n >= kMaxTimedLaunches) return;
  g_timer.name[g_timer.n] = name;
  cudaEventRecord(g_timer.ev[++g_timer.n], st);
}

template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(const char* name, void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
  if (e == cudaSuccess) timer_mark(name, st);
  return e;
}

// Limit of every in-kernel wait for another role's progress, for launches
// made by the current host thread (dsa_set_wait_limit_ns; default 2 s).
constexpr uint64_t kDefaultWaitLimitNs = 2000ull * 1000ull * 1000ull;
extern thread_local uint64_t g_wait_limit_ns;
__host__ inline uint64_t wait_limit_ns() { return g_wait_limit_ns; }

// Kernels launched by the current host thread since its last entry-point call
// began (reported by dsa_launches_in_last_call).
extern thread_local int g_launches;
__host__ inline cudaError_t counted(cudaError_t e) {
  if (e == cudaSuccess) ++g_launches;
  return e;
}


// Work plan written by k_plan (see k_prep.cu).
struct PlanBufs {
  int32_t* tok_seq;     // [T]
  int32_t* tok_pos;     // [T]
  int32_t* seq_gstart;  // [B+1]
  int4* groups;         // [max groups]  {b, t0, cnt, pos0}
  int4* items;          // [2 x max items] {b, t0, cnt, pos0}, {tile_begin, tile_end, g, 0}
  int32_t* counts;      // {groups, items}
};

// Tokens per indexer group and key tiles per work item for a geometry.
inline int indexer_group_tokens(int T, int B, bool fp8) { return T == B ? 1 : (fp8 ? 4 : 2); }
inline int indexer_item_tiles(int tg) { return tg == 1 ? 8 : 16; }
__host__ __device__ inline int64_t plan_max_groups(int T, int B, int tg) {
  const int64_t g = (int64_t)T / tg + B;
  return g < T ? g : T;
}
inline int64_t plan_max_items(int T, int B, int max_ctx, int tg) {
  const int64_t G = plan_max_groups(T, B, tg);
  const int64_t tiles = ((int64_t)max_ctx + 127) / 128;
  const int ch = indexer_item_tiles(tg);
  return G + (G * tiles + ch - 1) / ch;
}

// ---- launchers (each returns cudaGetLastError() of its launch) ----
cudaError_t launch_plan(const SeqsDev& s, int tg, int ch, const PlanBufs& p, uint32_t* err, cudaStream_t st);
// Plan + (FP8 / MXFP8 cache: qI quantization) + zeroing of `zero_words` words,
// one launch.  q_sf non-null selects MXFP8: the E8M0 group scales go to
// q_sf [T*64, 4].
cudaError_t launch_prep(const SeqsDev& s, int tg, int ch, const PlanBufs& plan, const __nv_bfloat16* qI,
                        const float* w, uint8_t* codes, float* w_scaled, uint8_t* q_sf, uint32_t* zero,
                        int64_t zero_words, uint32_t* err, cudaStream_t st);
cudaError_t launch_quantize_index_query(const __nv_bfloat16* qI, const float* w, int T, uint8_t* codes,
                                        float* w_scaled, cudaStream_t st);
cudaError_t launch_quantize_index_query_mx(const __nv_bfloat16* qI, int T, uint8_t* codes, uint8_t* scales,
                                           cudaStream_t st);
// Fused selection (decode): the indexer also selects the Top-K of every row
// (no score scratch).  Its grid is one CTA on each of kFusedGrid SMs, all
// resident; `tail` / `tail_items` (fused_topk_words words) start zeroed.
constexpr int kFusedGrid = 148;
constexpr int kFusedTailWordsPerToken = 2 * kTopkHistBins + 1024 + 8;  // 3 histograms, arrival counters
struct FusedTopk {
  uint32_t* tail;
  int2* tail_items;
  int2* cand;    // fused_topk_cand_bytes, need not be zeroed
  int32_t* idx;  // [T, K]
  int K;
};
int indexer_fused_capacity();                          // items per CTA
bool indexer_fused_fits(int T, int B, int max_ctx);    // the geometry fits the fused selection
int64_t fused_topk_words(int T, int B, int max_ctx);   // its zeroed scratch, in 32-bit words
size_t fused_topk_cand_bytes(int T);                   // its candidate lists
// Index-cache formats of the indexer kernel.
enum class IdxFmt { kBf16, kE4M3, kMx };
// E4M3 cache: codes/w_scaled from the quantizer, kI_scale fp32 [R];
// MXFP8 cache: codes and q_sf (E8M0 group scales) from the quantizer, w
// directly, kI_scale E8M0 bytes [R, 4]; bf16 cache: qI/w directly.
// hist (may be null; used for one token per group): Top-K first-digit histogram to accumulate into.
// fused (may be null): select the Top-K in the same kernel instead of writing scores.
cudaError_t launch_index_scores(const SeqsDev& s, const PlanBufs& plan, int tg, const void* q_operand,
                                const float* w_operand, const uint8_t* q_sf, const void* kI, const void* kI_scale,
                                IdxFmt fmt, float* scores, int64_t ld, uint32_t* hist, uint32_t* err,
                                cudaStream_t st, const FusedTopk* fused = nullptr);
size_t topk_scratch_bytes(int T, int64_t ld, int K);
// Several CTAs per row use a region at the head of the scratch that must be
// zero when they start (row counters + first-digit histogram, topk_zero_words
// words); `hist_ready` says the caller has zeroed it and filled the histogram.
bool topk_uses_hist(int T, int64_t ld);
int64_t topk_zero_words(int T);
uint32_t* topk_hist_in_scratch(void* scratch, int T);
cudaError_t launch_topk(const float* scores, int64_t ld, int T, const int32_t* row_len, const int32_t* tok_pos,
                        int K, int32_t* idx, void* scratch, bool hist_ready, uint32_t* err, cudaStream_t st);
size_t sparse_mla_partials_bytes(int T, int K, int H);
// kv: the bf16 pool, or (kv8_scale non-null) the FP8 cache's E4M3 codes with
// their tile-scale bytes [rows, 8].
cudaError_t launch_sparse_mla(const SeqsDev& s, TokenMap tm, bool tm_early, const __nv_bfloat16* q, const void* kv,
                              const uint8_t* kv8_scale, const int32_t* idx, int K, int H, float scale, void* out,
                              bool out_f32, float* lse, void* partials, uint32_t* err, cudaStream_t st);

}  // namespace dsa
