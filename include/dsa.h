/*
 * dsa.h -- C ABI of libdsa: index-selected sparse attention (DSA) on NVIDIA
 * B200 (sm_100a).
 *
 * The path has three stages, described (in prose, without a formula) by the
 * pages this library follows:
 *   [P1] "Day 0 Inference Adaptation and Performance Optimization for Hybrid
 *        Attention LLMs" -- Understanding the New Architecture, item 2
 *        ("Index-Selected Sparse Attention"), and Layer 1, "Sparse attention";
 *   [P2] "Hybrid Attention LLM Inference Acceleration: From Day-0 Support to
 *        Long-Sequence Performance Optimization" -- section 2 item 2 (indexer,
 *        sparse attention computation), section 4(1) (fused indexer reading the
 *        paged K cache), section 5 (quantized index Q/K);
 *   [P3] "Inference Acceleration for a New Domestic LLM Architecture..." --
 *        section 1 (LI and SFA) and section 3 (fused_lightning_indexer ->
 *        topk_select -> sparse_flash_attention pseudocode);
 *   [P4] "Optimizing Inference for Hybrid-Architecture Large Language
 *        Models..." -- section 2.2 and section 3.1 (three-in-one indexer);
 *   [P5] "Day-0 Inference Adaptation for Large Language Models..." --
 *        "Operator Fusion and Memory Access Optimization for Sparse Attention
 *        Paths" (Top-K indices passed straight to the compute kernel; paged KV).
 *
 * The exact formula implemented (the pages fix the stages, not the algebra):
 *   score[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])           s <= pos(t)
 *   S_t        = the min(K, pos(t)+1) positions with the largest score,
 *                equal scores -> lower position first
 *   out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . KV[s,0:576]) KV[s,0:512]
 *   lse[t,h]   = ln sum_{s in S_t} exp(scale * q[t,h,:] . KV[s,0:576])
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 * Sequences.  Sequence b holds ctx_len[b] cached tokens.  Its query tokens
 *   are the LAST q_len[b] = q_seq_start[b+1] - q_seq_start[b] of them, stored
 *   as rows q_seq_start[b] .. q_seq_start[b+1]-1 of every per-token tensor.
 *   Query j of sequence b sits at position pos = ctx_len[b] - q_len[b] + j and
 *   its candidates are positions 0..pos (the token itself included), so decode
 *   (q_len = 1), prefill (q_len = ctx) and chunked prefill share one form.
 * Paged pools.  Logical position s of sequence b lives in physical row
 *   page_table[b*max_pages + s/64]*64 + s%64 of each pool (page size 64).
 *   Pools: index keys kI [R, 128] (bf16; FP8 E4M3 codes with one fp32 scale
 *   per row in kI_scale [R]; or MXFP8: E4M3 codes with one E8M0 scale byte
 *   per 32 elements in kI_scale [R, 4]) and latent KV [R, 576] (bf16; or
 *   E4M3 codes with five power-of-two tile-scale bytes per row in
 *   kv_scale [R, 8], see dsa_kv_dtype_t), R = num_phys_pages*64.
 * Fixed sizes.  Index heads H_I = 64, index dim d_I = 128, latent dims
 *   576 (keys) / 512 (values), page size 64.  Attention heads H in {16, 32,
 *   64, 128}.  1 <= K <= 2048.  Anything else returns DSA_ERR_UNSUPPORTED.
 * Layouts.  Row-major, densely packed unless a leading dimension is given:
 *   qI [T,64,128] bf16, w [T,64] fp32, q [T,H,576] bf16, out [T,H,512] bf16,
 *   lse [T,H] fp32, idx [T,K] int32, scores [T,ld] fp32; out is bf16 or fp32
 *   (dsa_out_dtype_t).
 * Memory.  Every pointer argument is DEVICE memory owned by the caller; the
 *   library allocates nothing, keeps no state between calls and never
 *   synchronises the stream except inside dsa_check_error.  Device pointers
 *   must be 16-byte aligned; the paged pools 128-byte aligned.
 * Workspace.  ws is caller-owned device scratch of at least
 *   dsa_workspace_size(op, ...) bytes, 256-byte aligned, ZEROED ONCE before its
 *   first use (e.g. cudaMemset or torch.zeros).  Its first word is a sticky
 *   device error flag; calls that run concurrently must not share a workspace.
 * Errors.  Arguments are validated on the host before anything is launched;
 *   a failed check returns its status and launches nothing.  Values that only
 *   the device sees (lengths, page ids, indices) are bounds-checked in the
 *   kernels: a bad value is skipped (never dereferenced) and sets the error
 *   flag, which dsa_check_error() reports.  Kernels never trap.  Waits inside
 *   kernels are bounded; a wait that runs out sets DSA_ERR_TIMEOUT.
 * Execution.  All launches are asynchronous on `stream` (NULL = the legacy
 *   default stream).  Apart from dsa_check_error (which synchronises), the
 *   entry points make no synchronising or allocating CUDA call, so a CUDA
 *   graph can capture them.
 */
#ifndef DSA_H
#define DSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* An opaque cudaStream_t (struct CUstream_st*).  NULL = legacy default stream. */
typedef struct CUstream_st *dsa_stream_t;
/* An opaque cudaEvent_t (struct CUevent_st*). */
typedef struct CUevent_st *dsa_event_t;

typedef enum {
  DSA_OK = 0,
  DSA_ERR_INVALID_ARG = 1, /* null pointer, negative size, misaligned pointer  */
  DSA_ERR_UNSUPPORTED = 2, /* a size outside the fixed set listed above        */
  DSA_ERR_WORKSPACE = 3,   /* ws too small, null or not 256-byte aligned       */
  DSA_ERR_CUDA = 4,        /* a CUDA runtime call failed (launch error, ...)   */
  DSA_ERR_BAD_INDEX = 5,   /* device saw a bad length, page id or index        */
  DSA_ERR_TIMEOUT = 6      /* a bounded in-kernel wait ran out                 */
} dsa_status_t;

typedef enum {
  DSA_KI_BF16 = 0,     /* kI pool is bf16 [R,128]; kI_scale must be NULL         */
  DSA_KI_FP8_E4M3 = 1, /* kI pool is OCP E4M3 codes [R,128] + fp32 kI_scale [R] */
  DSA_KI_MXFP8 = 2     /* kI pool is OCP E4M3 codes [R,128] + E8M0 kI_scale
                          uint8 [R,4]: byte g scales elements 32g..32g+31 by
                          2^(byte - 127) ([P2] section 5 table, "Indexer Q/K":
                          MXFP8, one shared scale per group of 32; [P4] 4.2) */
} dsa_ki_dtype_t;

typedef enum {
  DSA_KV_BF16 = 0,     /* latent KV pool is bf16 [R,576]; kv_scale must be NULL   */
  DSA_KV_FP8_E4M3 = 1  /* latent KV pool is OCP E4M3 codes [R,576] + kv_scale uint8
                          [R,8]: byte j (j = 0..4) scales elements 128j..128j+127
                          (the last tile: the 64 rope dims) by 2^(byte - 127),
                          bytes 5..7 unused.  Bytes 1..254 are valid.  ([P2]
                          section 5 table, "Main attention KV cache": FP8, per
                          token-head tile of 128.)                              */
} dsa_kv_dtype_t;

typedef enum {
  DSA_OUT_BF16 = 0,    /* attention output stored as bf16 (rounded to nearest even) */
  DSA_OUT_F32 = 1      /* attention output stored as fp32 (no output rounding)      */
} dsa_out_dtype_t;

typedef enum {
  DSA_OP_QUANTIZE_INDEX_QUERY = 0,
  DSA_OP_INDEX_SCORES = 1,
  DSA_OP_TOPK = 2,
  DSA_OP_SPARSE_MLA = 3,
  DSA_OP_INDEX_TOPK_ATTN = 4,
  DSA_OP_INDEX_TOPK_ATTN_FUSED = 5  /* dsa_index_topk_attn_ex with DSA_SELECT_IN_INDEXER */
} dsa_op_t;

/* Flags of dsa_index_topk_attn_ex. */
enum {
  /* Decode batches (one query token per sequence) whose rows fit: the indexer
   * kernel selects the Top-K itself -- the fused scoring-weighting-selection
   * operator of [P2] section 4(1) / [P4] section 3.1 -- so no score array
   * exists and the call is at most four launches.  Workspace: size it with
   * DSA_OP_INDEX_TOPK_ATTN_FUSED.  Other geometries ignore the flag.  The
   * selected sets are the same as without it. */
  DSA_SELECT_IN_INDEXER = 1
};

/* Batch geometry (host struct; the three arrays are device memory).
 *   batch          B >= 1 sequences
 *   num_q_tokens   T = q_seq_start[B] >= 1 (host copy of the last entry)
 *   page_size      must be 64
 *   max_pages      columns of page_table, >= ceil(max_ctx / 64)
 *   num_phys_pages pages in each pool (R = 64 * num_phys_pages rows);
 *                  R above 2^31 - 1 returns DSA_ERR_UNSUPPORTED
 *   max_ctx        host-known upper bound of ctx_len[b]; sizes grids and
 *                  workspace.  A ctx_len above it is a device error.
 *   q_seq_start    int32 [B+1], non-decreasing, q_seq_start[0] = 0.  A
 *                  sequence whose rows leave 0..T-1 is skipped, and rows that
 *                  overlap (a decreasing entry) leave the indexer no work;
 *                  both are device errors (DSA_ERR_BAD_INDEX)
 *   ctx_len        int32 [B], q_len[b] <= ctx_len[b] <= max_ctx
 *   page_table     int32 [B, max_pages]; entries past ceil(ctx_len/64) unread
 */
typedef struct {
  int32_t batch;
  int32_t num_q_tokens;
  int32_t page_size;
  int32_t max_pages;
  int32_t num_phys_pages;
  int32_t max_ctx;
  const int32_t *q_seq_start;
  const int32_t *ctx_len;
  const int32_t *page_table;
} dsa_seqs_t;

/* Bytes of workspace `op` needs for this geometry, K and H (host only, no
 * CUDA call).  seqs->num_q_tokens and seqs->max_ctx are read; for DSA_OP_TOPK
 * pass num_q_tokens = rows and max_ctx = ld.  Returns 0 for invalid input. */
size_t dsa_workspace_size(dsa_op_t op, const dsa_seqs_t *seqs, int K, int H);

/* Index-query quantization, the indexer's input preparation ([P2] section 4(2)
 * "Q quantization"; [P3] section 3 `q_quantize`; format: [P2] section 5 table,
 * quantized index Q/K).  Per (token, head) row of qI: e = the smallest integer
 * with max|qI[t,h,:]| <= 448 * 2^e (e = 0 for a zero row); codes[t,h,:] =
 * E4M3(qI[t,h,:] / 2^e) rounded to nearest-even with saturation; w_scaled[t,h]
 * = w[t,h] * 2^e (the power-of-two scale folded into the head weight, exact).
 *   qI       bf16 [T,64,128]          codes     uint8 E4M3 [T,64,128] (out)
 *   w        fp32 [T,64]              w_scaled  fp32 [T,64] (out)
 * No workspace.  Errors: DSA_ERR_INVALID_ARG / DSA_ERR_CUDA. */
dsa_status_t dsa_quantize_index_query(const void *qI, const float *w, int T,
                                      uint8_t *codes, float *w_scaled,
                                      dsa_stream_t stream);

/* MXFP8 index-query quantization (the query side of DSA_KI_MXFP8; format:
 * [P2] section 5 table, "Indexer Q/K", one shared scale per group of 32;
 * [P4] section 4.2 per-group dynamic quantization).  For every group of 32
 * elements g of row (t,h): e = floor(log2(max |group|)) - 8 clamped to
 * [-127, 127] (e = 0 for an all-zero group); scales[t,h,g] = e + 127 (E8M0);
 * codes = E4M3(group / 2^e) rounded to nearest-even with saturation at 448.
 *   qI bf16 [T,64,128]; codes uint8 E4M3 [T,64,128] (out); scales uint8
 *   [T,64,4] (out).  No workspace.  Errors: DSA_ERR_INVALID_ARG / DSA_ERR_CUDA. */
dsa_status_t dsa_quantize_index_query_mx(const void *qI, int T, uint8_t *codes,
                                         uint8_t *scales, dsa_stream_t stream);

/* Lightweight-indexer scores ([P2] section 2 item 2 and section 4(1); [P3]
 * sections 1 and 3 `fused_lightning_indexer`; [P4] section 3.1): for every
 * query token t and candidate s = 0..pos(t),
 *   scores[t*ld + s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:]).
 * FP8 cache: kI[s] = E4M3(codes[s]) * kI_scale[s] and qI is first quantized as
 * in dsa_quantize_index_query (the scores are those of the quantized qI).
 * MXFP8 cache: kI[s,32g..32g+31] = E4M3(codes) * 2^(kI_scale[s,g] - 127) and qI
 * is first quantized as in dsa_quantize_index_query_mx; the group scales are
 * applied by the tensor core's block-scaled MMA.
 * Entries s > pos(t) of a row are left untouched.  ld >= max_ctx.
 * The reduction over heads happens in the kernel; no [T,H_I,N] tensor exists.
 *   qI bf16 [T,64,128]; w fp32 [T,64]; kI pool; kI_scale fp32 [R], uint8
 *   [R,4] (MXFP8) or NULL (bf16); scores fp32 [T,ld] (out). */
dsa_status_t dsa_index_scores(const dsa_seqs_t *seqs, const void *qI,
                              const float *w, const void *kI,
                              const void *kI_scale, dsa_ki_dtype_t ki_dtype,
                              float *scores, int64_t ld, void *ws,
                              size_t ws_bytes, dsa_stream_t stream);

/* Top-K selection ([P3] section 3 `topk_select`; [P2] section 2 item 2; [P4]
 * section 2.2 item 1).  Row t holds row_len[t] (device int32 [T]) valid scores
 * scores[t*ld + 0 .. row_len[t]-1].  idx[t*K + 0 ..] receives the positions of
 * the min(K, row_len[t]) largest scores -- equal scores prefer the lower
 * position, -0.0 equals +0.0 -- in ASCENDING order, padded with -1.  The
 * result is exactly determined (bit-exact).  NaN scores are not supported.
 * A row_len outside 0..ld sets DSA_ERR_BAD_INDEX (the row is clamped). */
dsa_status_t dsa_topk(const float *scores, int64_t ld, int T,
                      const int32_t *row_len, int K, int32_t *idx, void *ws,
                      size_t ws_bytes, dsa_stream_t stream);

/* Sparse MLA attention over selected positions ([P1] Understanding the New
 * Architecture item 2; [P2] section 2 item 2 "Sparse attention computation";
 * [P3] section 3 `sparse_flash_attention`; [P5] Operator Fusion, bullet 1:
 * the indices go straight into the compute kernel, no gathered copy exists).
 *   out[t,h,:] = sum_{s in idx[t]} softmax(scale * q[t,h,:] . KV[s,0:576]) KV[s,0:512]
 *   lse[t,h]   = natural-log sum-exp of the scaled logits (lse may be NULL).
 * idx [T,K] holds logical positions 0..pos(t) of token t's sequence, -1 =
 * unused slot, any order, no duplicates; at least one valid entry per row.
 * An entry outside -1..pos(t) sets DSA_ERR_BAD_INDEX and is skipped.
 *   q bf16 [T,H,576]; kv bf16 pool [R,576]; out [T,H,512] (out) of
 *   out_dtype (bf16 or fp32; the arithmetic is the same, fp32 accumulation). */
dsa_status_t dsa_sparse_mla_fwd(const dsa_seqs_t *seqs, const void *q,
                                const void *kv, const int32_t *idx, int K,
                                int H, float scale, void *out,
                                dsa_out_dtype_t out_dtype, float *lse,
                                void *ws, size_t ws_bytes, dsa_stream_t stream);

/* dsa_sparse_mla_fwd with the latent pool's format: kv_dtype DSA_KV_BF16
 * (kv_scale NULL) is dsa_sparse_mla_fwd; DSA_KV_FP8_E4M3 reads E4M3 codes kv
 * [R,576] and tile-scale bytes kv_scale [R,8] (16-byte aligned) and attends
 * over the dequantized rows KV[s,d] = E4M3(kv[s,d]) * 2^(kv_scale[s,d/128] - 127),
 * which are exact bf16 values, so the arithmetic is that of a bf16 pool
 * holding them.  Same workspace as dsa_sparse_mla_fwd. */
dsa_status_t dsa_sparse_mla_fwd_ex(const dsa_seqs_t *seqs, const void *q,
                                   const void *kv, const void *kv_scale,
                                   dsa_kv_dtype_t kv_dtype, const int32_t *idx,
                                   int K, int H, float scale, void *out,
                                   dsa_out_dtype_t out_dtype, float *lse,
                                   void *ws, size_t ws_bytes,
                                   dsa_stream_t stream);

/* Size of the scratch array dsa_sparse_mla_fwd_noalloc uses (32 MiB). */
#define DSA_NOALLOC_SCRATCH_BYTES (32u << 20)

/* dsa_sparse_mla_fwd for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry point: it serves code that only ever
 * receives input and output buffers -- a plugin inside a host framework that
 * owns every device allocation, or a caller running where cudaMalloc is not
 * permitted -- and so has nothing to pass as `ws`.
 * Inputs, outputs and results are those of dsa_sparse_mla_fwd.  The scratch is
 * a fixed array of DSA_NOALLOC_SCRATCH_BYTES in the library's device image:
 *   - every GPU that loads the library holds that memory until the process exits;
 *   - a geometry whose scratch (dsa_workspace_size(DSA_OP_SPARSE_MLA, ...))
 *     exceeds it returns DSA_ERR_WORKSPACE before any CUDA call (a batch whose
 *     index lists are split over several CTAs -- fewer than 148 (token, 64-head
 *     group) pairs -- needs at most ~20 MiB; larger batches need only 8 bytes
 *     per token plus 4 per sequence);
 *   - each call looks up the array's device address in the current context
 *     (a host-side runtime query; the device must be current);
 *   - nothing is allocated or freed (no cudaMalloc, cudaFree or allocating
 *     library routine); the array's error word is cleared at the start of each
 *     call with an asynchronous memset;
 *   - all calls share the one array, which keeps the last call's contents:
 *     calls that overlap on the GPU (other streams, other host threads) race
 *     and corrupt each other's results, so serialise them;
 *   - bad device-side indices or page ids are skipped as in dsa_sparse_mla_fwd,
 *     and a bounded in-kernel wait that runs out abandons its slice, whose
 *     partial result the merge may then take from an earlier call; both set the
 *     array's error word, which only dsa_check_error_noalloc reads: call it
 *     after the call (before the next one) to know the result is sound. */
dsa_status_t dsa_sparse_mla_fwd_noalloc(const dsa_seqs_t *seqs, const void *q,
                                        const void *kv, const int32_t *idx,
                                        int K, int H, float scale, void *out,
                                        dsa_out_dtype_t out_dtype, float *lse,
                                        dsa_stream_t stream);

/* dsa_check_error for dsa_sparse_mla_fwd_noalloc: synchronises `stream`, then
 * reads and clears the error word of the built-in scratch array (the device
 * must be current).  Same results as dsa_check_error. */
dsa_status_t dsa_check_error_noalloc(dsa_stream_t stream);

/* The whole path in one call ([P1] Layer 1, "Sparse attention": scoring,
 * selection, gathering and attention integrated; [P3] section 3 pseudocode):
 * dsa_index_scores -> dsa_topk -> dsa_sparse_mla_fwd on the caller's stream,
 * with the scores and indices living in the workspace.  idx_out (may be NULL)
 * receives the selected positions [T,K] as dsa_topk returns them. */
dsa_status_t dsa_index_topk_attn(const dsa_seqs_t *seqs, const void *qI,
                                 const float *w, const void *kI,
                                 const void *kI_scale, dsa_ki_dtype_t ki_dtype,
                                 const void *q, const void *kv, int K, int H,
                                 float scale, void *out,
                                 dsa_out_dtype_t out_dtype, float *lse,
                                 int32_t *idx_out, void *ws, size_t ws_bytes,
                                 dsa_stream_t stream);

/* dsa_index_topk_attn with options.  `kv_scale` / `kv_dtype`: the latent
 * pool's format, as in dsa_sparse_mla_fwd_ex.  `flags`: 0 or DSA_SELECT_IN_INDEXER.
 * `q_ready`: for a caller whose attention query q is still being
 * produced or copied on another stream when the call is made ([P2] section
 * 4(2): the indexer's inputs are prepared apart from the attention's, so the
 * two overlap).  Everything up to the attention stage is launched at once;
 * the attention launch first waits on `q_ready` (cudaStreamWaitEvent on
 * `stream`), so q must hold its final values when the event completes.
 * q_ready NULL is dsa_index_topk_attn.  The event must have been recorded
 * before the call. */
dsa_status_t dsa_index_topk_attn_ex(const dsa_seqs_t *seqs, const void *qI,
                                    const float *w, const void *kI,
                                    const void *kI_scale, dsa_ki_dtype_t ki_dtype,
                                    const void *q, const void *kv,
                                    const void *kv_scale, dsa_kv_dtype_t kv_dtype,
                                    int K, int H, float scale, void *out,
                                    dsa_out_dtype_t out_dtype, float *lse,
                                    int32_t *idx_out, void *ws, size_t ws_bytes,
                                    unsigned flags, dsa_event_t q_ready,
                                    dsa_stream_t stream);

/* Synchronises `stream`, reads and clears the workspace's sticky device error
 * flag.  Returns DSA_OK, DSA_ERR_BAD_INDEX, DSA_ERR_TIMEOUT or DSA_ERR_CUDA
 * (a pending CUDA error on the stream). */
dsa_status_t dsa_check_error(void *ws, dsa_stream_t stream);

/* Limit, in nanoseconds, of every bounded in-kernel wait for another part of
 * the kernel to make progress, for the launches of later calls made by the
 * calling host thread (0 restores the default of 2 s).  A wait that runs out
 * sets DSA_ERR_TIMEOUT and its CTA winds down (waiting, under a fixed 2 s
 * bound, only for copies and MMAs it has already issued).  A failure-handling
 * aid: a short limit makes waits run out on purpose.  Host only; DSA_OK. */
dsa_status_t dsa_set_wait_limit_ns(uint64_t ns);

/* Number of kernels the calling host thread's most recent entry-point call
 * (dsa_quantize_index_query .. dsa_index_topk_attn) launched.  Host only. */
int dsa_launches_in_last_call(void);

/* Per-launch device timing: a measurement aid with no counterpart in the
 * method's description.  enable != 0: every later entry-point call made by the
 * calling host thread records a CUDA event on its stream before its first
 * kernel and one after each kernel it launches -- so each kernel then runs
 * without overlapping its neighbours, and the call is slower than untimed.
 * enable == 0 stops this and destroys the events.  The events belong to the
 * device current at the enabling call (thread-local library state, the one
 * exception to "no state between calls").  Returns DSA_OK or DSA_ERR_CUDA. */
dsa_status_t dsa_launch_timing(int enable);

/* For the calling thread's most recent entry-point call made with timing on:
 * waits for its last event, then writes up to `cap` entries -- ms[i], the
 * device milliseconds from the event before kernel i to the one after it, and
 * names[i], a static string naming the kernel (either array may be NULL).
 * Returns how many kernels that call launched (possibly more than cap; at
 * most 16 are timed), 0 if timing was off for it, -1 on a CUDA error. */
int dsa_last_launch_times(float *ms, const char **names, int cap);

/* Static, human-readable name of a status. */
const char *dsa_status_string(dsa_status_t status);

#ifdef __cplusplus
}
#endif
#endif /* DSA_H */
