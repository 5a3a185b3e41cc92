// Host side of the C ABI declared in include/dsa.h: argument validation,
// workspace layout and the launch sequence of each entry point.  Nothing here
// allocates, synchronises (except dsa_check_error) or reads device memory.
#include <cmath>

#include "dsa_internal.cuh"

using namespace dsa;

namespace dsa {
thread_local int g_launches = 0;
thread_local LaunchTimer g_timer;
thread_local uint64_t g_wait_limit_ns = kDefaultWaitLimitNs;
}

namespace {

constexpr size_t kAlign = 256;
size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

// Workspace carve-up.  Offsets are 256-byte aligned; the first 256 bytes hold
// the sticky error word.
struct Layout {
  size_t tok_seq = 0, tok_pos = 0, seq_gstart = 0, groups = 0, items = 0, counts = 0;
  size_t q_codes = 0, w_scaled = 0, q_sf = 0, scores = 0, idx = 0, topk = 0, partials = 0, tail = 0, cand = 0;
  size_t total = 0;
  int64_t ld = 0;
  bool fused = false;       // the indexer selects the Top-K itself (no score scratch)
  int64_t tail_words = 0;
};

// The indexer's work-list capacity must hold for either index-cache dtype, so
// it is sized for the smaller group (more groups, more items).
int sizing_group_tokens(int T, int B) { return T == B ? 1 : 2; }

Layout make_layout(dsa_op_t op, int T, int B, int max_ctx, int K, int H) {
  Layout L;
  size_t off = kAlign;  // header: the sticky error word
  auto take = [&](size_t bytes) {
    size_t o = off;
    off = align_up(off + bytes);
    return o;
  };
  const bool fused_op = op == DSA_OP_INDEX_TOPK_ATTN_FUSED;
  if (fused_op) op = DSA_OP_INDEX_TOPK_ATTN;  // the same call, its selection inside the indexer when the rows fit
  const bool seq_ops = op == DSA_OP_INDEX_SCORES || op == DSA_OP_SPARSE_MLA || op == DSA_OP_INDEX_TOPK_ATTN;
  const bool indexer = op == DSA_OP_INDEX_SCORES || op == DSA_OP_INDEX_TOPK_ATTN;
  if (seq_ops) {
    L.tok_seq = take((size_t)T * sizeof(int32_t));
    L.tok_pos = take((size_t)T * sizeof(int32_t));
    L.seq_gstart = take((size_t)(B + 1) * sizeof(int32_t));
    L.counts = take(4 * sizeof(int32_t));
  }
  if (indexer) {
    const int tg = sizing_group_tokens(T, B);
    L.groups = take((size_t)plan_max_groups(T, B, tg) * sizeof(int4));
    L.items = take((size_t)plan_max_items(T, B, max_ctx, tg) * 2 * sizeof(int4));
    L.q_codes = take((size_t)T * kHI * kDI);
    L.w_scaled = take((size_t)T * kHI * sizeof(float));
    L.q_sf = take((size_t)T * kHI * 4);  // MXFP8 query group scales (E8M0)
  }
  if (op == DSA_OP_INDEX_TOPK_ATTN) {
    L.ld = ((int64_t)max_ctx + 3) / 4 * 4;
    L.fused = fused_op && indexer_fused_fits(T, B, max_ctx);
    if (L.fused) {  // decode: selection inside the indexer, its histograms and counts only
      L.tail_words = fused_topk_words(T, B, max_ctx);
      L.tail = take((size_t)L.tail_words * sizeof(uint32_t));
      L.cand = take(fused_topk_cand_bytes(T));
      L.idx = take((size_t)T * K * sizeof(int32_t));
    } else {
      L.scores = take((size_t)T * (size_t)L.ld * sizeof(float));
      L.idx = take((size_t)T * K * sizeof(int32_t));
      L.topk = take(topk_scratch_bytes(T, L.ld, K));
    }
  }
  if (op == DSA_OP_TOPK) L.topk = take(topk_scratch_bytes(T, max_ctx, K));
  if (op == DSA_OP_SPARSE_MLA || op == DSA_OP_INDEX_TOPK_ATTN) L.partials = take(sparse_mla_partials_bytes(T, K, H));
  L.total = off;
  return L;
}

template <class T>
T* at(void* ws, size_t off) {
  return reinterpret_cast<T*>(reinterpret_cast<char*>(ws) + off);
}

bool valid_H(int H) { return H == 16 || H == 32 || H == 64 || H == 128; }

dsa_status_t check_seqs(const dsa_seqs_t* s) {
  if (!s || !s->q_seq_start || !s->ctx_len || !s->page_table) return DSA_ERR_INVALID_ARG;
  if (s->batch < 1 || s->num_q_tokens < 1 || s->max_ctx < 1 || s->num_phys_pages < 1 || s->max_pages < 1)
    return DSA_ERR_INVALID_ARG;
  if (s->page_size != kPage) return DSA_ERR_UNSUPPORTED;
  if ((int64_t)s->max_pages * kPage < (int64_t)s->max_ctx) return DSA_ERR_INVALID_ARG;
  // pool rows are 32-bit in the kernels (TMA coordinates, gathered row ids)
  if ((int64_t)s->num_phys_pages * kPage > (int64_t)INT32_MAX) return DSA_ERR_UNSUPPORTED;
  return DSA_OK;
}

dsa_status_t check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (!ws || !aligned(ws, kAlign) || ws_bytes < need) return DSA_ERR_WORKSPACE;
  return DSA_OK;
}

SeqsDev to_dev(const dsa_seqs_t* s) {
  SeqsDev d;
  d.batch = s->batch;
  d.num_tokens = s->num_q_tokens;
  d.max_pages = s->max_pages;
  d.num_phys_pages = s->num_phys_pages;
  d.max_ctx = s->max_ctx;
  d.q_seq_start = s->q_seq_start;
  d.ctx_len = s->ctx_len;
  d.page_table = s->page_table;
  return d;
}

dsa_status_t cuda_status(cudaError_t e) { return e == cudaSuccess ? DSA_OK : DSA_ERR_CUDA; }

#define DSA_TRY(x)                       \
  do {                                   \
    dsa_status_t _st = (x);              \
    if (_st != DSA_OK) return _st;       \
  } while (0)
#define DSA_CUDA(x) DSA_TRY(cuda_status(x))

dsa_status_t check_indexer_args(const dsa_seqs_t* seqs, const void* qI, const float* w, const void* kI,
                                const void* kI_scale, dsa_ki_dtype_t ki_dtype) {
  DSA_TRY(check_seqs(seqs));
  if (!qI || !w || !kI) return DSA_ERR_INVALID_ARG;
  if (ki_dtype != DSA_KI_BF16 && ki_dtype != DSA_KI_FP8_E4M3 && ki_dtype != DSA_KI_MXFP8) return DSA_ERR_UNSUPPORTED;
  if ((ki_dtype != DSA_KI_BF16) != (kI_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (!aligned(qI, 16) || !aligned(w, 16) || !aligned(kI, 128) || (kI_scale && !aligned(kI_scale, 16)))
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa_status_t check_kv_args(const void* kv_scale, dsa_kv_dtype_t kv_dtype) {
  if (kv_dtype != DSA_KV_BF16 && kv_dtype != DSA_KV_FP8_E4M3) return DSA_ERR_UNSUPPORTED;
  if ((kv_dtype == DSA_KV_FP8_E4M3) != (kv_scale != nullptr)) return DSA_ERR_INVALID_ARG;
  if (kv_scale && !aligned(kv_scale, 16)) return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

dsa_status_t check_attn_args(const dsa_seqs_t* seqs, const void* q, const void* kv, int K, int H, float scale,
                             const void* out, dsa_out_dtype_t out_dtype, const float* lse) {
  DSA_TRY(check_seqs(seqs));
  if (out_dtype != DSA_OUT_BF16 && out_dtype != DSA_OUT_F32) return DSA_ERR_UNSUPPORTED;
  if (!q || !kv || !out) return DSA_ERR_INVALID_ARG;
  if (K < 1 || K > kMaxK || !valid_H(H)) return DSA_ERR_UNSUPPORTED;
  if (!std::isfinite(scale)) return DSA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(kv, 128) || !aligned(out, 16) || (lse && !aligned(lse, 4)))
    return DSA_ERR_INVALID_ARG;
  return DSA_OK;
}

PlanBufs plan_bufs(void* ws, const Layout& L) {
  PlanBufs p;
  p.tok_seq = at<int32_t>(ws, L.tok_seq);
  p.tok_pos = at<int32_t>(ws, L.tok_pos);
  p.seq_gstart = at<int32_t>(ws, L.seq_gstart);
  p.groups = L.groups ? at<int4>(ws, L.groups) : nullptr;
  p.items = L.items ? at<int4>(ws, L.items) : nullptr;
  p.counts = at<int32_t>(ws, L.counts);
  return p;
}

// Tokens per indexer group for a call: one for decode, else two (bf16 and
// MXFP8 caches) or four (E4M3 cache).
int group_tokens(const dsa_seqs_t* seqs, dsa_ki_dtype_t ki_dtype) {
  return indexer_group_tokens(seqs->num_q_tokens, seqs->batch, ki_dtype == DSA_KI_FP8_E4M3);
}

// Indexer launch sequence shared by dsa_index_scores and the fused call: one
// prep launch (plan, FP8 / MXFP8 query quantization, zeroing of `zero`) and
// the indexer, which also accumulates Top-K's first-digit histogram into
// `hist` when that is given (one token per group).
dsa_status_t run_indexer(const dsa_seqs_t* seqs, const SeqsDev& sd, const PlanBufs& plan, int tg, const void* qI,
                         const float* w, const void* kI, const void* kI_scale, dsa_ki_dtype_t ki_dtype,
                         float* scores, int64_t ld, void* ws, const Layout& L, uint32_t* hist, uint32_t* zero,
                         int64_t zero_words, uint32_t* err, cudaStream_t st, const FusedTopk* fused = nullptr) {
  const bool fp8 = ki_dtype == DSA_KI_FP8_E4M3, mx = ki_dtype == DSA_KI_MXFP8;
  const void* q_operand = qI;
  const float* w_operand = w;
  uint8_t* codes = (fp8 || mx) ? at<uint8_t>(ws, L.q_codes) : nullptr;
  float* w_scaled = fp8 ? at<float>(ws, L.w_scaled) : nullptr;
  uint8_t* q_sf = mx ? at<uint8_t>(ws, L.q_sf) : nullptr;
  DSA_CUDA(launch_prep(sd, tg, indexer_item_tiles(tg), plan,
                       (fp8 || mx) ? reinterpret_cast<const __nv_bfloat16*>(qI) : nullptr, w, codes, w_scaled, q_sf,
                       zero, zero_words, err, st));
  if (fp8) {
    q_operand = codes;
    w_operand = w_scaled;
  } else if (mx) {
    q_operand = codes;  // the head weights stay as given: the group scales ride in the MMA
  }
  const IdxFmt fmt = mx ? IdxFmt::kMx : (fp8 ? IdxFmt::kE4M3 : IdxFmt::kBf16);
  DSA_CUDA(launch_index_scores(sd, plan, tg, q_operand, w_operand, q_sf, kI, kI_scale, fmt, scores, ld, hist, err, st,
                               fused));
  return DSA_OK;
}

}  // namespace

extern "C" {

size_t dsa_workspace_size(dsa_op_t op, const dsa_seqs_t* seqs, int K, int H) {
  if (!seqs || seqs->num_q_tokens < 1 || seqs->max_ctx < 1) return 0;
  if (op == DSA_OP_QUANTIZE_INDEX_QUERY) return 0;
  if (op == DSA_OP_TOPK) return make_layout(op, seqs->num_q_tokens, 1, seqs->max_ctx, K, 16).total;
  if (op < 0 || op > DSA_OP_INDEX_TOPK_ATTN_FUSED) return 0;
  if (seqs->batch < 1) return 0;
  if ((op == DSA_OP_SPARSE_MLA || op == DSA_OP_INDEX_TOPK_ATTN || op == DSA_OP_INDEX_TOPK_ATTN_FUSED) &&
      (K < 1 || K > kMaxK || !valid_H(H)))
    return 0;
  return make_layout(op, seqs->num_q_tokens, seqs->batch, seqs->max_ctx, K, H).total;
}

dsa_status_t dsa_quantize_index_query(const void* qI, const float* w, int T, uint8_t* codes, float* w_scaled,
                                      dsa_stream_t stream) {
  g_launches = 0;
  if (!qI || !w || !codes || !w_scaled || T < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned(qI, 16) || !aligned(codes, 16) || !aligned(w, 4) || !aligned(w_scaled, 4))
    return DSA_ERR_INVALID_ARG;
  timer_begin((cudaStream_t)stream);
  return cuda_status(launch_quantize_index_query(reinterpret_cast<const __nv_bfloat16*>(qI), w, T, codes, w_scaled,
                                                 (cudaStream_t)stream));
}

dsa_status_t dsa_quantize_index_query_mx(const void* qI, int T, uint8_t* codes, uint8_t* scales,
                                         dsa_stream_t stream) {
  g_launches = 0;
  if (!qI || !codes || !scales || T < 1) return DSA_ERR_INVALID_ARG;
  if (!aligned(qI, 16) || !aligned(codes, 16) || !aligned(scales, 4)) return DSA_ERR_INVALID_ARG;
  timer_begin((cudaStream_t)stream);
  return cuda_status(launch_quantize_index_query_mx(reinterpret_cast<const __nv_bfloat16*>(qI), T, codes, scales,
                                                    (cudaStream_t)stream));
}

dsa_status_t dsa_index_scores(const dsa_seqs_t* seqs, const void* qI, const float* w, const void* kI,
                              const void* kI_scale, dsa_ki_dtype_t ki_dtype, float* scores, int64_t ld, void* ws,
                              size_t ws_bytes, dsa_stream_t stream) {
  g_launches = 0;
  DSA_TRY(check_indexer_args(seqs, qI, w, kI, kI_scale, ki_dtype));
  if (!scores || ld < seqs->max_ctx || !aligned(scores, 16)) return DSA_ERR_INVALID_ARG;
  const Layout L = make_layout(DSA_OP_INDEX_SCORES, seqs->num_q_tokens, seqs->batch, seqs->max_ctx, 1, 16);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* err = at<uint32_t>(ws, 0);
  const SeqsDev sd = to_dev(seqs);
  const PlanBufs plan = plan_bufs(ws, L);
  const int tg = group_tokens(seqs, ki_dtype);
  timer_begin(st);
  return run_indexer(seqs, sd, plan, tg, qI, w, kI, kI_scale, ki_dtype, scores, ld, ws, L, nullptr, nullptr, 0, err,
                     st);
}

dsa_status_t dsa_topk(const float* scores, int64_t ld, int T, const int32_t* row_len, int K, int32_t* idx, void* ws,
                      size_t ws_bytes, dsa_stream_t stream) {
  g_launches = 0;
  if (!scores || !row_len || !idx || T < 1 || ld < 1) return DSA_ERR_INVALID_ARG;
  if (K < 1 || K > kMaxK) return DSA_ERR_UNSUPPORTED;
  if (ld > INT32_MAX) return DSA_ERR_UNSUPPORTED;
  if (!aligned(scores, 16) || !aligned(row_len, 4) || !aligned(idx, 16)) return DSA_ERR_INVALID_ARG;
  const Layout L = make_layout(DSA_OP_TOPK, T, 1, (int)ld, K, 16);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  timer_begin((cudaStream_t)stream);
  return cuda_status(
      launch_topk(scores, ld, T, row_len, nullptr, K, idx, at<void>(ws, L.topk), false, at<uint32_t>(ws, 0),
                  (cudaStream_t)stream));
}

dsa_status_t dsa_sparse_mla_fwd_ex(const dsa_seqs_t* seqs, const void* q, const void* kv, const void* kv_scale,
                                   dsa_kv_dtype_t kv_dtype, const int32_t* idx, int K, int H, float scale, void* out,
                                   dsa_out_dtype_t out_dtype, float* lse, void* ws, size_t ws_bytes,
                                   dsa_stream_t stream) {
  g_launches = 0;
  DSA_TRY(check_attn_args(seqs, q, kv, K, H, scale, out, out_dtype, lse));
  DSA_TRY(check_kv_args(kv_scale, kv_dtype));
  if (!idx || !aligned(idx, 16)) return DSA_ERR_INVALID_ARG;
  const Layout L = make_layout(DSA_OP_SPARSE_MLA, seqs->num_q_tokens, seqs->batch, seqs->max_ctx, K, H);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* err = at<uint32_t>(ws, 0);
  const SeqsDev sd = to_dev(seqs);
  const PlanBufs plan = plan_bufs(ws, L);
  TokenMap tm{plan.tok_seq, plan.tok_pos};
  timer_begin(st);
  DSA_CUDA(launch_plan(sd, 1, 0, plan, err, st));  // token geometry only
  DSA_CUDA(launch_sparse_mla(sd, tm, /*tm_early=*/false, reinterpret_cast<const __nv_bfloat16*>(q), kv,
                             static_cast<const uint8_t*>(kv_scale), idx, K, H, scale, out,
                             out_dtype == DSA_OUT_F32, lse, at<void>(ws, L.partials), err, st));
  return DSA_OK;
}

dsa_status_t dsa_sparse_mla_fwd(const dsa_seqs_t* seqs, const void* q, const void* kv, const int32_t* idx, int K,
                                int H, float scale, void* out, dsa_out_dtype_t out_dtype, float* lse, void* ws,
                                size_t ws_bytes, dsa_stream_t stream) {
  return dsa_sparse_mla_fwd_ex(seqs, q, kv, nullptr, DSA_KV_BF16, idx, K, H, scale, out, out_dtype, lse, ws, ws_bytes,
                               stream);
}

dsa_status_t dsa_index_topk_attn_ex(const dsa_seqs_t* seqs, const void* qI, const float* w, const void* kI,
                                    const void* kI_scale, dsa_ki_dtype_t ki_dtype, const void* q, const void* kv,
                                    const void* kv_scale, dsa_kv_dtype_t kv_dtype, int K,
                                    int H, float scale, void* out, dsa_out_dtype_t out_dtype, float* lse,
                                    int32_t* idx_out, void* ws, size_t ws_bytes, unsigned flags,
                                    dsa_event_t q_ready, dsa_stream_t stream) {
  g_launches = 0;
  DSA_TRY(check_indexer_args(seqs, qI, w, kI, kI_scale, ki_dtype));
  DSA_TRY(check_attn_args(seqs, q, kv, K, H, scale, out, out_dtype, lse));
  DSA_TRY(check_kv_args(kv_scale, kv_dtype));
  if (idx_out && !aligned(idx_out, 16)) return DSA_ERR_INVALID_ARG;
  if (flags & ~(unsigned)DSA_SELECT_IN_INDEXER) return DSA_ERR_INVALID_ARG;
  const Layout L = make_layout((flags & DSA_SELECT_IN_INDEXER) ? DSA_OP_INDEX_TOPK_ATTN_FUSED : DSA_OP_INDEX_TOPK_ATTN,
                               seqs->num_q_tokens, seqs->batch, seqs->max_ctx, K, H);
  DSA_TRY(check_ws(ws, ws_bytes, L.total));
  cudaStream_t st = (cudaStream_t)stream;
  uint32_t* err = at<uint32_t>(ws, 0);
  const SeqsDev sd = to_dev(seqs);
  const PlanBufs plan = plan_bufs(ws, L);
  TokenMap tm{plan.tok_seq, plan.tok_pos};
  int32_t* idx = idx_out ? idx_out : at<int32_t>(ws, L.idx);
  const int T = seqs->num_q_tokens;
  const int tg = group_tokens(seqs, ki_dtype);
  if (L.fused) {
    // decode: prep, the indexer with the Top-K selection inside, attention
    uint32_t* tail = at<uint32_t>(ws, L.tail);
    const FusedTopk f{tail, reinterpret_cast<int2*>(tail + (size_t)T * kFusedTailWordsPerToken),
                      at<int2>(ws, L.cand), idx, K};
    timer_begin(st);
    DSA_TRY(run_indexer(seqs, sd, plan, tg, qI, w, kI, kI_scale, ki_dtype, nullptr, L.ld, ws, L, nullptr, tail,
                        L.tail_words, err, st, &f));
    if (q_ready) DSA_CUDA(cudaStreamWaitEvent(st, (cudaEvent_t)q_ready, 0));
    DSA_CUDA(launch_sparse_mla(sd, tm, /*tm_early=*/true, reinterpret_cast<const __nv_bfloat16*>(q), kv,
                               static_cast<const uint8_t*>(kv_scale), idx, K, H, scale,
                               out, out_dtype == DSA_OUT_F32, lse, at<void>(ws, L.partials), err, st));
    return DSA_OK;
  }
  float* scores = at<float>(ws, L.scores);
  // one token per group: the indexer also builds Top-K's first-digit histogram
  const bool fuse_hist = tg == 1 && topk_uses_hist(T, L.ld);
  uint32_t* hist = fuse_hist ? topk_hist_in_scratch(at<void>(ws, L.topk), T) : nullptr;
  uint32_t* zero = fuse_hist ? at<uint32_t>(ws, L.topk) : nullptr;  // Top-K's counters + histogram
  timer_begin(st);
  DSA_TRY(run_indexer(seqs, sd, plan, tg, qI, w, kI, kI_scale, ki_dtype, scores, L.ld, ws, L, hist, zero,
                      fuse_hist ? topk_zero_words(T) : 0, err, st));
  DSA_CUDA(launch_topk(scores, L.ld, T, nullptr, tm.pos, K, idx, at<void>(ws, L.topk), hist != nullptr, err, st));
  // the query may still be in flight on another stream: attention is the first step that reads it
  if (q_ready) DSA_CUDA(cudaStreamWaitEvent(st, (cudaEvent_t)q_ready, 0));
  DSA_CUDA(launch_sparse_mla(sd, tm, /*tm_early=*/true, reinterpret_cast<const __nv_bfloat16*>(q), kv,
                             static_cast<const uint8_t*>(kv_scale), idx, K, H, scale,
                             out, out_dtype == DSA_OUT_F32, lse, at<void>(ws, L.partials), err, st));
  return DSA_OK;
}

dsa_status_t dsa_index_topk_attn(const dsa_seqs_t* seqs, const void* qI, const float* w, const void* kI,
                                 const void* kI_scale, dsa_ki_dtype_t ki_dtype, const void* q, const void* kv, int K,
                                 int H, float scale, void* out, dsa_out_dtype_t out_dtype, float* lse,
                                 int32_t* idx_out, void* ws, size_t ws_bytes, dsa_stream_t stream) {
  return dsa_index_topk_attn_ex(seqs, qI, w, kI, kI_scale, ki_dtype, q, kv, nullptr, DSA_KV_BF16, K, H, scale, out,
                                out_dtype, lse, idx_out, ws, ws_bytes, 0u, nullptr, stream);
}

dsa_status_t dsa_check_error(void* ws, dsa_stream_t stream) {
  if (!ws) return DSA_ERR_WORKSPACE;
  cudaStream_t st = (cudaStream_t)stream;
  if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  uint32_t flag = 0;
  if (cudaMemcpy(&flag, ws, sizeof(flag), cudaMemcpyDeviceToHost) != cudaSuccess) return DSA_ERR_CUDA;
  if (flag) {
    if (cudaMemsetAsync(ws, 0, sizeof(flag), st) != cudaSuccess) return DSA_ERR_CUDA;
    if (cudaStreamSynchronize(st) != cudaSuccess) return DSA_ERR_CUDA;
  }
  if (flag & kErrTimeout) return DSA_ERR_TIMEOUT;
  if (flag & kErrBadIndex) return DSA_ERR_BAD_INDEX;
  return DSA_OK;
}

int dsa_launches_in_last_call(void) { return g_launches; }

dsa_status_t dsa_set_wait_limit_ns(uint64_t ns) {
  g_wait_limit_ns = ns == 0 ? kDefaultWaitLimitNs : ns;
  return DSA_OK;
}

dsa_status_t dsa_launch_timing(int enable) {
  LaunchTimer& tm = g_timer;
  if (tm.device >= 0) {  // tear down (also before re-enabling)
    int cur = -1;
    cudaGetDevice(&cur);
    if (cur != tm.device) cudaSetDevice(tm.device);
    for (cudaEvent_t& e : tm.ev) {
      if (e) cudaEventDestroy(e);
      e = nullptr;
    }
    if (cur >= 0 && cur != tm.device) cudaSetDevice(cur);
    tm.device = -1;
  }
  tm.armed = false;
  tm.n = 0;
  if (!enable) return DSA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return DSA_ERR_CUDA;
  for (cudaEvent_t& e : tm.ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      e = nullptr;
      for (cudaEvent_t& f : tm.ev) {  // release the ones already made: timing stays off
        if (f) cudaEventDestroy(f);
        f = nullptr;
      }
      return DSA_ERR_CUDA;
    }
  }
  tm.device = dev;
  return DSA_OK;
}

int dsa_last_launch_times(float* ms, const char** names, int cap) {
  const LaunchTimer& tm = g_timer;
  if (!tm.armed || tm.n == 0) return 0;
  if (cudaEventSynchronize(tm.ev[tm.n]) != cudaSuccess) return -1;
  for (int i = 0; i < tm.n && i < cap; ++i) {
    if (ms && cudaEventElapsedTime(&ms[i], tm.ev[i], tm.ev[i + 1]) != cudaSuccess) return -1;
    if (names) names[i] = tm.name[i];
  }
  return g_launches > tm.n ? g_launches : tm.n;
}

const char* dsa_status_string(dsa_status_t s) {
  switch (s) {
    case DSA_OK: return "DSA_OK";
    case DSA_ERR_INVALID_ARG: return "DSA_ERR_INVALID_ARG";
    case DSA_ERR_UNSUPPORTED: return "DSA_ERR_UNSUPPORTED";
    case DSA_ERR_WORKSPACE: return "DSA_ERR_WORKSPACE";
    case DSA_ERR_CUDA: return "DSA_ERR_CUDA";
    case DSA_ERR_BAD_INDEX: return "DSA_ERR_BAD_INDEX";
    case DSA_ERR_TIMEOUT: return "DSA_ERR_TIMEOUT";
  }
  return "DSA_ERR_UNKNOWN";
}

}  // extern "C"
