"""Helpers shared by the GPU parity tests: oracle runs on the generator's
bytes and the comparison rules of the library's accuracy contract.

Tolerances (written here once, used by every GPU test):
  * dsa_topk on given fp32 scores: index arrays bit-exact;
  * indexer scores: per row, max_s |gpu - ref| <= 1e-2 * rms_s(ref)  (the FP8
    path is judged against the oracle on the same quantized query);
  * end-to-end selection: every position in the symmetric difference of the
    GPU and oracle index sets has |ref_score - tau| <= 1e-3 * |tau|, tau = the
    oracle's K-th largest score of the row; rows with n <= K must match exactly;
  * attention output: max |gpu - ref| <= 1e-2 * rms(ref) over the whole output
    for fp32 output; a bf16 output may in addition differ by the half ulp of
    bf16 at |ref| that storing in bf16 costs (that rounding belongs to the
    output format: with max|out| above ~2.5 rms it alone exceeds 1e-2 rms);
    lse: |gpu - ref| <= 1e-3 * max(1, |ref|).
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import dsa_oracle as O
from dsa_workloads import Workload, bits16

SCORE_TOL = 1e-2
TIE_TOL = 1e-3
OUT_TOL = 1e-2
LSE_TOL = 1e-3


def oracle_seqs(wl: Workload) -> O.Seqs:
    return O.Seqs(ctx_len=wl.ctx_len.astype(np.int64), q_seq_start=wl.q_seq_start.astype(np.int64),
                  page_table=wl.page_table, page_size=wl.spec.page_size)


def kI_host(wl: Workload):
    if wl.kI_scale is None:
        return bits16(wl.kI), None
    return wl.kI.numpy(), wl.kI_scale.numpy()


def kv_host(wl: Workload):
    """The latent pool as the oracle takes it: bf16 bit patterns, or the FP8
    cache's (codes, scale bytes)."""
    if wl.kv_scale is None:
        return bits16(wl.kv)
    return wl.kv.numpy(), wl.kv_scale.numpy()


def oracle_scores(wl: Workload, tokens=None):
    kI, sc = kI_host(wl)
    return O.index_scores(oracle_seqs(wl), bits16(wl.qI), wl.w.numpy(), kI, sc, tokens=tokens)


def sample_tokens(wl: Workload, n: int, seed: int = 0) -> np.ndarray:
    """First, last, the rows around n_t = K, and a seeded sample."""
    T = wl.T
    pos = wl.token_pos()
    picks = {0, T - 1}
    K = wl.spec.topk
    near = np.nonzero(np.abs(pos + 1 - K) <= 1)[0]
    picks |= set(int(x) for x in near[:6])
    rng = np.random.default_rng(seed)
    picks |= set(int(x) for x in rng.choice(T, size=min(n, T), replace=False))
    return np.array(sorted(picks))


def assert_scores_close(gpu_rows, ref_rows, tokens):
    for t, g, r in zip(tokens, gpu_rows, ref_rows):
        rms = float(np.sqrt(np.mean(r * r)))
        err = float(np.max(np.abs(g.astype(np.float64) - r)))
        assert err <= SCORE_TOL * max(rms, 1e-30), f"token {t}: max err {err:.3e} vs rms {rms:.3e}"


def selection_violations(gpu_idx_row, ref_row, K):
    """Positions in the symmetric difference that are not near-ties of tau."""
    n = ref_row.shape[0]
    g = set(int(x) for x in gpu_idx_row if x >= 0)
    ref_idx = O.topk_select(ref_row, K)
    r = set(int(x) for x in ref_idx if x >= 0)
    if n <= K:
        return sorted(g ^ r)
    order = np.sort(ref_row)[::-1]
    tau = order[K - 1]
    bad = [s for s in (g ^ r) if not (0 <= s < n) or abs(ref_row[s] - tau) > TIE_TOL * abs(tau)]
    if len(g) != min(K, n):
        bad.append(-999)
    return bad


def bf16_half_ulp(x):
    a = np.abs(np.asarray(x, np.float64))
    e = np.floor(np.log2(np.maximum(a, 2.0 ** -126)))
    return np.exp2(e - 8)


def assert_attention_close(gpu_out, gpu_lse, ref_out, ref_lse):
    ref_out = np.asarray(ref_out)
    g = gpu_out.float().cpu().numpy().astype(np.float64)
    rms = float(np.sqrt(np.mean(ref_out * ref_out)))
    diff = np.abs(g - ref_out)
    if gpu_out.dtype == torch.float32:
        err = float(diff.max())
        assert err <= OUT_TOL * rms, f"attention (fp32 out) max err {err:.3e} vs rms {rms:.3e}"
    else:
        excess = diff - bf16_half_ulp(ref_out)
        err = float(excess.max())
        assert err <= OUT_TOL * rms, f"attention (bf16 out) max err beyond half-ulp {err:.3e} vs rms {rms:.3e}"
    if gpu_lse is not None:
        gl = gpu_lse.cpu().numpy().astype(np.float64)
        lerr = np.abs(gl - ref_lse) / np.maximum(1.0, np.abs(ref_lse))
        assert float(lerr.max()) <= LSE_TOL, f"lse err {float(lerr.max()):.3e}"


def device_rows(scores: torch.Tensor, wl: Workload, tokens):
    pos = wl.token_pos()
    host = scores.cpu().numpy()
    return [host[t, : pos[t] + 1] for t in tokens]


def topk_idx_for(wl: Workload, ref_rows, tokens):
    """Oracle index list [T, K] (rows not in tokens left -1)."""
    idx = np.full((wl.T, wl.spec.topk), -1, np.int32)
    for t, r in zip(tokens, ref_rows):
        idx[t] = O.topk_select(r, wl.spec.topk)
    return idx
