"""Plain fp64 CPU oracle for index-selected sparse attention (DSA).

TEST INFRASTRUCTURE ONLY.  The library never imports, links or calls anything
here; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may.  It shares no code, header, table or constant generator with
the CUDA path: the only thing both sides see is the seeded synthetic input
(``dsa_workloads``), which holds none of the method's
arithmetic.

Sources.  Five web pages describe one engineering effort on DSA; they are cited
by title and section:

  [P1] "Day 0 Inference Adaptation and Performance Optimization for Hybrid
       Attention LLMs"
  [P2] "Hybrid Attention LLM Inference Acceleration: From Day-0 Support to
       Long-Sequence Performance Optimization"
  [P3] "Inference Acceleration for a New Domestic LLM Architecture: From Day-0
       Adaptation to Full-Pipeline Performance Optimization"
  [P4] "Optimizing Inference for Hybrid-Architecture Large Language Models: From
       Operator Fusion to Layer-Aware Quantization"
  [P5] "Day-0 Inference Adaptation for Large Language Models: Technical
       Approaches and Practical Insights"

The pages name the stages (indexer scoring, head-weight weighting, Top-K over
a paged K cache, sparse reads of the latent KV) but print no formula.  The
library's specification fixes it, and this module writes it out literally:

    score[t,s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:])          s <= pos(t)
    S_t        = the K positions with the largest score; ties -> lower s
    out[t,h,:] = sum_{s in S_t} softmax_s(scale * q[t,h,:] . KV[s,0:576]) * KV[s,0:512]

Readings taken where the pages are silent (each repeated at its function):
  * candidates of query t are the positions 0..pos(t), the token itself
    included (the indexer scores every earlier position: [P1] Understanding
    the New Architecture item 2; [P2] §2 item 2);
  * a row with fewer than K candidates takes all of them, index list padded
    with -1, and the selected indices are emitted in ascending order;
  * the FP8 index cache is OCP E4M3 with one fp32 scale per token row; the bf16
    index query is quantized per (token, head) with a power-of-two scale;
  * MXFP8 (the pages' index format: one shared scale per group of 32) is read
    as the OCP Microscaling format: E4M3 elements sharing an E8M0 power-of-two
    scale per block of 32, the scale 2^(floor(log2 amax) - 8), elements of the
    block's top binade above 448 saturating.  Cache and query both take it;
  * the FP8 latent KV cache (the pages: FP8, per token-head tile of 128) cuts
    each 576-value latent row into tiles of 128 (the last, the 64 rope dims,
    of 64) with one power-of-two scale per tile, the tightest that needs no
    saturation (so every dequantized value is an exact bf16 number).

Every function here is pinned by a test in ``tests/test_oracle_*.py`` against
something other than itself (library routines, brute force, closed forms,
invariants, a hand-expanded example).  No function is "parity unpinned".
All arithmetic is float64 on the exact values the GPU consumes.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

# ----------------------------------------------------------------------------
# Number formats
# ----------------------------------------------------------------------------


def bf16_to_f64(bits) -> np.ndarray:
    """Exact value of bfloat16 bit patterns (the top half of an IEEE binary32)."""
    b = np.asarray(bits, dtype=np.uint16)
    with np.errstate(invalid="ignore"):  # NaN patterns widen to NaN
        return (b.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def e4m3_decode(codes) -> np.ndarray:
    """Exact value of OCP FP8 E4M3 codes: 1 sign bit, 4 exponent bits (bias 7),
    3 mantissa bits; exponent 0 is subnormal (m * 2^-9); S.1111.111 is NaN and
    there is no infinity, so the largest finite magnitude is 1.75 * 2^8 = 448.
    The FP8 format of the index cache: [P2] §5 table ("Indexer Q/K"), [P4] §4.1.
    """
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    sign = np.where(c & 0x80, -1.0, 1.0)
    e = (c >> 3) & 0xF
    m = (c & 0x7).astype(np.float64)
    mag = np.where(e == 0, m * 2.0 ** -9, (1.0 + m / 8.0) * np.exp2(e.astype(np.float64) - 7.0))
    mag = np.where((e == 15) & (c & 0x7 == 7), np.nan, mag)
    return sign * mag


# The 127 non-negative finite E4M3 values, code 0x00 .. 0x7E, strictly increasing.
_E4M3_NONNEG = e4m3_decode(np.arange(0x7F, dtype=np.uint8))
E4M3_MAX = 448.0
# Lookup for decoding large arrays fast (same values as e4m3_decode).
_E4M3_LUT = e4m3_decode(np.arange(256, dtype=np.uint8))


def e4m3_decode_fast(codes) -> np.ndarray:
    return _E4M3_LUT[np.asarray(codes, dtype=np.uint8)]


def e4m3_encode(x) -> np.ndarray:
    """Round real values to E4M3 codes: nearest representable value, ties to the
    code with an even mantissa (round-to-nearest-even), magnitudes at or above
    448 saturate to 448 ("satfinite"), the sign is kept (so tiny negatives give
    -0), NaN gives 0x7F.
    """
    x = np.asarray(x, dtype=np.float64)
    a = np.abs(x)
    i = np.clip(np.searchsorted(_E4M3_NONNEG, a, side="right") - 1, 0, 126)
    lo = _E4M3_NONNEG[i]
    hi = _E4M3_NONNEG[np.minimum(i + 1, 126)]
    d_lo = a - lo
    d_hi = hi - a
    round_up = (d_lo > d_hi) | ((d_lo == d_hi) & (i % 2 == 1))
    code = np.where(round_up, i + 1, i)
    code = np.where(a >= E4M3_MAX, 126, code)
    code = code | np.where(np.signbit(x), 0x80, 0)
    code = np.where(np.isnan(x), 0x7F, code)
    return code.astype(np.uint8)


# ----------------------------------------------------------------------------
# Index-query quantization  ([P2] §4(2): "Q quantization" is one of the indexer's
# input-preparation steps; [P3] §3 pseudocode `q_quantize`; [P4] §3.2)
# ----------------------------------------------------------------------------


def pow2_exponent(amax: float) -> int:
    """Smallest integer e with amax <= 448 * 2^e (0 when amax == 0).

    The scale 2^e is the power-of-two analogue of amax/448: dividing by it maps
    the row into the E4M3 range without saturation and is exact in binary.
    """
    amax = float(amax)
    if amax == 0.0:
        return 0
    e = math.ceil(math.log2(amax / E4M3_MAX))
    while amax > E4M3_MAX * 2.0 ** e:
        e += 1
    while amax <= E4M3_MAX * 2.0 ** (e - 1):
        e -= 1
    return e


def quantize_index_query(qI_bits):
    """bf16 index query [T, H_I, d_I] -> (E4M3 codes [T, H_I, d_I], scale [T, H_I]).

    One power-of-two scale per (token, head) row: sq = 2^e with e from
    ``pow2_exponent(max |q|)``; codes = E4M3(q / sq).  Reading: the pages quantize
    the index Q ([P2] §5 table; [P3] §4) with group scales; per-row pow2 scaling
    is the plainest format that keeps the whole head row in one FP8 MMA operand.
    """
    q = bf16_to_f64(qI_bits)
    amax = np.abs(q).max(axis=-1)
    e = np.vectorize(pow2_exponent, otypes=[np.int64])(amax)
    sq = np.exp2(e.astype(np.float64))
    codes = e4m3_encode(q / sq[..., None])
    return codes, sq


# ----------------------------------------------------------------------------
# MXFP8 ([P2] §5 table, "Indexer Q/K": MXFP8 dynamic quantization, per group of
# 32 elements sharing one scale factor; [P3] §4 "Layered Quantization"; [P4]
# §4.2 "Per-Group Dynamic Quantization")
# ----------------------------------------------------------------------------

MX_BLOCK = 32        # elements sharing one scale
E8M0_BIAS = 127
E4M3_EMAX = 8        # exponent of E4M3's top binade: 448 = 1.75 * 2^8


def e8m0_decode(codes) -> np.ndarray:
    """Exact value of E8M0 scale codes: 2^(code - 127), code 255 is NaN.  E8M0
    (8 exponent bits, no sign, no mantissa) is the shared-scale format of the
    OCP Microscaling formats, of which MXFP8 is the E4M3 member."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    v = np.ldexp(1.0, c - E8M0_BIAS)
    return np.where(c == 255, np.nan, v)


def mx_shared_exponent(amax: float) -> int:
    """Exponent e of one block's scale 2^e: floor(log2(amax)) - 8, so that the
    block's largest magnitude lands in E4M3's top binade [256, 512); clamped to
    E8M0's range [-127, 127].  An all-zero block takes e = 0 (reading: the
    format leaves it open, and any scale encodes zeros)."""
    amax = float(amax)
    if amax == 0.0:
        return 0
    _, ex = math.frexp(amax)           # amax = m * 2^ex, 0.5 <= m < 1: floor(log2 amax) = ex - 1
    return int(min(127, max(-127, ex - 1 - E4M3_EMAX)))


def mxfp8_quantize(x):
    """Real values [..., n] (n a multiple of 32) -> (E4M3 codes [..., n],
    E8M0 scale codes [..., n/32]).  Block i covers elements 32i .. 32i+31 of
    the last axis; codes = E4M3(x / 2^e) rounded to nearest-even and saturated
    at +-448 (``e4m3_encode``), e = ``mx_shared_exponent(max |block|)``."""
    x = np.asarray(x, dtype=np.float64)
    n = x.shape[-1]
    if n % MX_BLOCK:
        raise ValueError("the last axis must be a multiple of 32")
    blocks = x.reshape(*x.shape[:-1], n // MX_BLOCK, MX_BLOCK)
    amax = np.abs(blocks).max(axis=-1)
    e = np.vectorize(mx_shared_exponent, otypes=[np.int64])(amax)
    codes = e4m3_encode(blocks / np.ldexp(1.0, e)[..., None])
    return codes.reshape(x.shape), (e + E8M0_BIAS).astype(np.uint8)


def mxfp8_dequantize(codes, scales) -> np.ndarray:
    """Exact value of MXFP8 data: E4M3(codes) * 2^(scale - 127) per block of 32."""
    c = np.asarray(codes, dtype=np.uint8)
    n = c.shape[-1]
    v = e4m3_decode_fast(c).reshape(*c.shape[:-1], n // MX_BLOCK, MX_BLOCK)
    return (v * e8m0_decode(scales)[..., None]).reshape(c.shape)


# ----------------------------------------------------------------------------
# FP8 latent KV cache ([P2] §5 table, "Main attention KV cache": FP8, per
# token-head tile, tile size 128; [P3] §4 "Layered Quantization")
# ----------------------------------------------------------------------------

KV_TILE = 128        # elements per scale along the latent row
KV_SCALE_COLS = 8    # scale bytes stored per row: one per tile (5 used), zero padding


def kv_fp8_quantize(kv):
    """Real latent rows [R, 576] -> (E4M3 codes [R, 576], scale bytes [R, 8]).

    Tile j holds elements 128j .. 128j+127 of the row (tile 4: the 64 rope
    dims 512..575).  Its scale is 2^e with e = ``pow2_exponent(max |tile|)``,
    the smallest power of two for which nothing saturates; codes = E4M3(x / 2^e)
    rounded to nearest-even; byte j of the row's scales holds e + 127, bytes
    5..7 are 0.  Reading: the pages fix the granularity, not the scale format;
    a power-of-two scale keeps every dequantized value an exact bf16 number."""
    x = np.asarray(kv, dtype=np.float64)
    R, D = x.shape
    ntiles = (D + KV_TILE - 1) // KV_TILE
    codes = np.zeros((R, D), dtype=np.uint8)
    scales = np.zeros((R, KV_SCALE_COLS), dtype=np.uint8)
    for j in range(ntiles):
        lo, hi = j * KV_TILE, min(D, (j + 1) * KV_TILE)
        amax = np.abs(x[:, lo:hi]).max(axis=1)
        e = np.vectorize(pow2_exponent, otypes=[np.int64])(amax)
        codes[:, lo:hi] = e4m3_encode(x[:, lo:hi] / np.ldexp(1.0, e)[:, None])
        scales[:, j] = (e + E8M0_BIAS).astype(np.uint8)
    return codes, scales


def kv_fp8_dequantize(codes, scales) -> np.ndarray:
    """Exact values of FP8 latent rows: E4M3(codes) * 2^(scale byte - 127) per tile."""
    c = np.asarray(codes, dtype=np.uint8)
    sc = np.asarray(scales, dtype=np.uint8)
    v = e4m3_decode_fast(c).copy()
    for j in range((c.shape[-1] + KV_TILE - 1) // KV_TILE):
        lo, hi = j * KV_TILE, min(c.shape[-1], (j + 1) * KV_TILE)
        v[..., lo:hi] *= e8m0_decode(sc[..., j])[..., None]
    return v


def kv_rows(kv, rows) -> np.ndarray:
    """Exact values of latent-pool rows `rows`: the pool is bf16 bit patterns
    [R, 576] (uint16), or an FP8 cache given as (codes [R, 576], scales [R, 8])."""
    if isinstance(kv, tuple):
        codes, scales = kv
        return kv_fp8_dequantize(np.asarray(codes)[rows], np.asarray(scales)[rows])
    return bf16_to_f64(np.asarray(kv)[rows])


def is_mx_scale(kI_scale) -> bool:
    """An MXFP8 index cache carries E8M0 codes [R, 4] (uint8); an E4M3 cache one
    fp32 scale per row."""
    return kI_scale is not None and np.asarray(kI_scale).dtype == np.uint8


# ----------------------------------------------------------------------------
# Sequences and the paged caches
# ([P2] §2 item 2: the indexer reads the paged K cache directly;
#  [P5] "Operator Fusion and Memory Access Optimization for Sparse Attention
#  Paths": KV blocks under paged management)
# ----------------------------------------------------------------------------


@dataclass
class Seqs:
    """Batch geometry.  Sequence b holds ctx_len[b] cached tokens; its query
    tokens are the last q_len[b] of them, stored as rows q_seq_start[b] ..
    q_seq_start[b+1]-1 of every per-token tensor.  Logical position s of
    sequence b lives in physical row page_table[b, s // page_size] * page_size
    + s % page_size of each pool."""

    ctx_len: np.ndarray       # int [B]
    q_seq_start: np.ndarray   # int [B+1]
    page_table: np.ndarray    # int [B, max_pages]
    page_size: int

    @property
    def num_tokens(self) -> int:
        return int(self.q_seq_start[-1])

    def token_seq_pos(self, t: int):
        """(sequence, absolute position) of query token t."""
        b = int(np.searchsorted(self.q_seq_start, t, side="right") - 1)
        q_len = int(self.q_seq_start[b + 1] - self.q_seq_start[b])
        pos = int(self.ctx_len[b]) - q_len + (t - int(self.q_seq_start[b]))
        return b, pos

    def rows(self, b: int, positions) -> np.ndarray:
        """Physical pool rows of logical positions of sequence b."""
        s = np.asarray(positions, dtype=np.int64)
        pages = self.page_table[b][s // self.page_size].astype(np.int64)
        if np.any(pages < 0):
            raise ValueError("position maps to an unassigned page")
        return pages * self.page_size + s % self.page_size


def _token_list(seqs: Seqs, tokens):
    return range(seqs.num_tokens) if tokens is None else [int(t) for t in tokens]


# ----------------------------------------------------------------------------
# Stage 1: lightweight indexer scores
# ([P1] Understanding the New Architecture item 2; [P2] §2 item 2 "Indexer";
#  [P3] §1 and §3; [P4] §2.2 item 1 and §3.1)
# ----------------------------------------------------------------------------


def index_scores(seqs: Seqs, qI_bits, w, kI, kI_scale=None, tokens=None):
    """Indexer score of every causal candidate of each query token.

    score[t, s] = sum_h w[t,h] * ReLU(qI[t,h,:] . kI[s,:]),  s = 0 .. pos(t).

    bf16 index cache (``kI_scale is None``): qI and kI are the bf16 values.
    FP8 index cache: kI[s] = E4M3(codes[s]) * kI_scale[s] (per-token scale) and
    qI is replaced by its quantized form E4M3(q^)[t,h] * sq[t,h]
    (``quantize_index_query``); since sq, kI_scale > 0 the ReLU commutes with
    them, so the score is  kI_scale[s] * sum_h w[t,h] sq[t,h] ReLU(q^ . k^).
    MXFP8 index cache (kI_scale = E8M0 codes [R, 4], ``is_mx_scale``): kI[s] =
    ``mxfp8_dequantize(codes[s], kI_scale[s])`` and each (token, head) row of
    qI is replaced by ``mxfp8_dequantize(*mxfp8_quantize(row))``; the scores
    are the formula above on those values.

    Returns a list with one float64 array of length pos(t)+1 per token
    (in the order of ``tokens``; all tokens when None).
    """
    w = np.asarray(w, dtype=np.float64)
    mx = is_mx_scale(kI_scale)
    fp8 = kI_scale is not None and not mx
    if mx:
        qvals = mxfp8_dequantize(*mxfp8_quantize(bf16_to_f64(qI_bits)))
    elif fp8:
        qhat, sq = quantize_index_query(qI_bits)
        qvals = e4m3_decode_fast(qhat)
    else:
        qvals = bf16_to_f64(qI_bits)
    out = []
    for t in _token_list(seqs, tokens):
        b, pos = seqs.token_seq_pos(t)
        rows = seqs.rows(b, np.arange(pos + 1))
        if mx:
            kmat = mxfp8_dequantize(np.asarray(kI)[rows], np.asarray(kI_scale)[rows])
            wt = w[t]
        elif fp8:
            kmat = e4m3_decode_fast(np.asarray(kI)[rows])
            wt = w[t] * sq[t]
        else:
            kmat = bf16_to_f64(np.asarray(kI)[rows])
            wt = w[t]
        dots = qvals[t] @ kmat.T                      # [H_I, n]
        score = wt @ np.maximum(dots, 0.0)            # [n]
        if fp8:
            score = score * np.asarray(kI_scale, dtype=np.float64)[rows]
        out.append(score)
    return out


# ----------------------------------------------------------------------------
# Stage 2: Top-K selection
# ([P3] §3 pseudocode `topk_select`; [P2] §2 item 2; [P4] §2.2 item 1)
# ----------------------------------------------------------------------------


def topk_select(scores_row, K: int) -> np.ndarray:
    """Positions of the min(K, n) largest scores of one row.

    Order of preference: larger score first, equal scores -> lower position
    first; -0.0 and +0.0 are equal.  The chosen positions are returned in
    ascending order, padded with -1 to length K.  NaN scores are not a valid
    input (they cannot arise from finite inputs) and raise.
    """
    s = np.asarray(scores_row, dtype=np.float64) + 0.0   # x + 0.0 maps -0.0 to +0.0
    if np.isnan(s).any():
        raise ValueError("NaN score")
    n = s.shape[0]
    order = np.lexsort((np.arange(n), -s))             # primary: -score, then position
    chosen = np.sort(order[: min(K, n)])
    out = np.full(K, -1, dtype=np.int32)
    out[: chosen.shape[0]] = chosen
    return out


def topk_rows(rows, K: int) -> np.ndarray:
    return np.stack([topk_select(r, K) for r in rows]) if len(rows) else np.zeros((0, K), np.int32)


# ----------------------------------------------------------------------------
# Stage 3: sparse MLA attention over the selected latent rows
# ([P1] Understanding the New Architecture item 2: attention over low-rank
#  compressed (latent) KV reading only the selected positions; [P2] §1 (MLA) and
#  §2 item 2 "Sparse attention computation"; [P3] §1 and §3
#  `sparse_flash_attention`; [P4] §2.2 item 2)
# ----------------------------------------------------------------------------


def sparse_mla(seqs: Seqs, q_bits, kv_bits, idx, scale: float, d_v: int = 512, tokens=None):
    """out[t,h,:] = sum_{s in S_t} p_s KV[s, 0:d_v],
    p = softmax_s(scale * q[t,h,:] . KV[s, :]),  lse[t,h] = ln sum_s exp(scale * logit).

    Keys are the whole latent row (latent + rope, 576 values); values are its
    first d_v = 512 (the latent).  All heads share the KV rows.  idx[t] holds
    logical positions with -1 padding; the order of idx does not matter.
    kv_bits: the bf16 pool, or an FP8 cache (codes, scales) (``kv_rows``).
    Returns (out [n_tok, H, d_v], lse [n_tok, H]) in float64.
    """
    idx = np.asarray(idx)
    tl = list(_token_list(seqs, tokens))
    H = np.asarray(q_bits).shape[1]
    out = np.zeros((len(tl), H, d_v))
    lse = np.zeros((len(tl), H))
    for i, t in enumerate(tl):
        b, pos = seqs.token_seq_pos(t)
        sel = idx[t][idx[t] >= 0].astype(np.int64)
        if sel.size == 0 or sel.max() > pos or np.unique(sel).size != sel.size:
            raise ValueError(f"token {t}: invalid selection")
        kmat = kv_rows(kv_bits, seqs.rows(b, sel))                    # [k, 576]
        qt = bf16_to_f64(np.asarray(q_bits)[t])                       # [H, 576]
        logits = scale * (qt @ kmat.T)                                # [H, k]
        m = logits.max(axis=1, keepdims=True)
        p = np.exp(logits - m)
        l = p.sum(axis=1, keepdims=True)
        out[i] = (p @ kmat[:, :d_v]) / l
        lse[i] = (m + np.log(l))[:, 0]
    return out, lse


def dense_masked_mla(seqs: Seqs, q_bits, kv_bits, scale: float, d_v: int = 512, tokens=None):
    """Dense causal attention over every position 0..pos(t) (no selection).

    Written with its own loop structure (per head, explicit two-pass softmax,
    masking of positions beyond pos with -inf over the whole context) so that
    ``sparse_mla`` with K >= context can be checked against it.
    """
    tl = list(_token_list(seqs, tokens))
    q_bits = np.asarray(q_bits)
    H = q_bits.shape[1]
    out = np.zeros((len(tl), H, d_v))
    lse = np.zeros((len(tl), H))
    for i, t in enumerate(tl):
        b, pos = seqs.token_seq_pos(t)
        ctx = int(seqs.ctx_len[b])
        full = np.empty((ctx, np.asarray(kv_bits).shape[1]))
        for s in range(ctx):          # gather the sequence's whole logical K row by row
            page = int(seqs.page_table[b, s // seqs.page_size])
            full[s] = bf16_to_f64(np.asarray(kv_bits)[page * seqs.page_size + s % seqs.page_size])
        for h in range(H):
            qh = bf16_to_f64(q_bits[t, h])
            logit = np.full(ctx, -np.inf)
            logit[: pos + 1] = scale * (full[: pos + 1] @ qh)
            mx = np.max(logit)
            e = np.exp(logit - mx)                                 # masked entries give 0
            den = e.sum()
            out[i, h] = (e[:, None] * full[:, :d_v]).sum(axis=0) / den
            lse[i, h] = mx + math.log(den)
    return out, lse


# ----------------------------------------------------------------------------
# The whole path ([P3] §3 pseudocode: indexer -> topk_select -> sparse attention;
# [P1] Layer 1 "Sparse attention" bullet: scoring, selection, gathering, compute)
# ----------------------------------------------------------------------------


def index_topk_attn(seqs: Seqs, qI_bits, w, kI, kI_scale, q_bits, kv_bits, K: int,
                    scale: float, d_v: int = 512, tokens=None):
    """Composition of the three stages.  Returns (scores, idx, out, lse) for
    ``tokens`` (all when None); idx rows are in the order of ``tokens``."""
    tl = list(_token_list(seqs, tokens))
    scores = index_scores(seqs, qI_bits, w, kI, kI_scale, tokens=tl)
    idx_rows = topk_rows(scores, K)
    full_idx = np.full((seqs.num_tokens, K), -1, dtype=np.int32)
    for i, t in enumerate(tl):
        full_idx[t] = idx_rows[i]
    out, lse = sparse_mla(seqs, q_bits, kv_bits, full_idx, scale, d_v=d_v, tokens=tl)
    return scores, idx_rows, out, lse
