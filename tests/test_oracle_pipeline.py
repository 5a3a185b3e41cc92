"""Pins of the oracle's whole path (indexer -> Top-K -> sparse MLA, composed by
``index_topk_attn``) that do not restate it:

* with K at least the context every causal candidate is kept, so the result is
  the dense causal masked attention whatever the index scores are;
* with K = 1 and one planted key per query token that dominates its index score,
  Top-K must return that position and attention over a single key is that key's
  value row, with lse = scale * q . k;
* the rows of a call over a subset of tokens (in any order) are the rows of the
  call over all tokens.
"""
import math

import numpy as np
import torch

from oracle import dsa_oracle as O

H_I, D_I, H, DQK, DV, PS = 2, 8, 3, 12, 8, 4


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _geometry(rng, B, prefill):
    ctx = rng.integers(3, 15, B)
    q_len = ctx.copy() if prefill else np.ones(B, np.int64)
    pages = (ctx + PS - 1) // PS
    n_pages = int(pages.sum()) + 2
    perm = rng.permutation(n_pages)
    pt = np.full((B, pages.max()), -1, np.int32)
    k = 0
    for b in range(B):
        pt[b, : pages[b]] = perm[k: k + pages[b]]
        k += pages[b]
    qs = np.concatenate([[0], np.cumsum(q_len)])
    return O.Seqs(ctx_len=ctx, q_seq_start=qs, page_table=pt, page_size=PS), n_pages * PS


def _inputs(rng, seqs, R):
    T = seqs.num_tokens
    qI = rng.standard_normal((T, H_I, D_I))
    w = rng.standard_normal((T, H_I))
    kI = rng.standard_normal((R, D_I))
    q = rng.standard_normal((T, H, DQK))
    kv = rng.standard_normal((R, DQK))
    return _bf16_bits(qI), w, _bf16_bits(kI), _bf16_bits(q), _bf16_bits(kv)


def test_all_candidates_kept_gives_dense_attention():
    rng = np.random.default_rng(21)
    for prefill in (True, False):
        seqs, R = _geometry(rng, 3, prefill)
        qI, w, kI, q, kv = _inputs(rng, seqs, R)
        scale = 1.0 / math.sqrt(DQK)
        _, idx, out, lse = O.index_topk_attn(seqs, qI, w, kI, None, q, kv, 16, scale, d_v=DV)
        for t in range(seqs.num_tokens):
            _, pos = seqs.token_seq_pos(t)
            assert np.array_equal(idx[t], np.r_[np.arange(pos + 1), np.full(16 - pos - 1, -1)])
        d_out, d_lse = O.dense_masked_mla(seqs, q, kv, scale, d_v=DV)
        assert np.allclose(out, d_out, rtol=1e-12, atol=1e-12)
        assert np.allclose(lse, d_lse, rtol=1e-12, atol=1e-12)


def test_planted_key_with_k1_reduces_to_its_value_row():
    rng = np.random.default_rng(22)
    seqs, R = _geometry(rng, 4, prefill=False)   # one query token per sequence
    T = seqs.num_tokens
    qI = np.ones((T, H_I, D_I))
    w = np.abs(rng.standard_normal((T, H_I))) + 0.5
    kI = rng.standard_normal((R, D_I)) * 0.01
    planted = []
    for t in range(T):
        b, pos = seqs.token_seq_pos(t)
        s = int(rng.integers(0, pos + 1))
        kI[seqs.rows(b, [s])[0]] = 10.0             # index score 80 * sum(w) against |.| < 1 elsewhere
        planted.append((b, s))
    q = _bf16_bits(rng.standard_normal((T, H, DQK)))
    kv = _bf16_bits(rng.standard_normal((R, DQK)))
    scale = 0.37
    _, idx, out, lse = O.index_topk_attn(seqs, _bf16_bits(qI), w, _bf16_bits(kI), None, q, kv, 1, scale, d_v=DV)
    for t, (b, s) in enumerate(planted):
        assert idx[t].tolist() == [s]
        kvec = (kv[seqs.rows(b, [s])[0]].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        qmat = (q[t].astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        for h in range(H):
            assert np.array_equal(out[t, h], kvec[:DV])
            ref = scale * math.fsum(qmat[h, d] * kvec[d] for d in range(DQK))
            assert math.isclose(lse[t, h], ref, rel_tol=1e-12, abs_tol=1e-12)


def test_token_subset_gives_the_same_rows():
    rng = np.random.default_rng(23)
    seqs, R = _geometry(rng, 3, prefill=True)
    qI, w, kI, q, kv = _inputs(rng, seqs, R)
    K, scale = 5, 0.25
    full = O.index_topk_attn(seqs, qI, w, kI, None, q, kv, K, scale, d_v=DV)
    T = seqs.num_tokens
    sub = [T - 1, 0, T // 2]
    part = O.index_topk_attn(seqs, qI, w, kI, None, q, kv, K, scale, d_v=DV, tokens=sub)
    for i, t in enumerate(sub):
        assert np.array_equal(part[0][i], full[0][t])
        assert np.array_equal(part[1][i], full[1][t])
        assert np.allclose(part[2][i], full[2][t], rtol=1e-13, atol=1e-13)
        assert np.allclose(part[3][i], full[3][t], rtol=1e-13, atol=1e-13)
