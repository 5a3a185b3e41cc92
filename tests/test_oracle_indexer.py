"""Pins of the oracle's indexer: the hand-expanded 4-token example (bf16 and FP8
cache forms), invariances of the paged layout and the scaling laws of the
formula."""
import json
import os

import numpy as np
import torch

from oracle import dsa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden", "indexer_hand_4tok.json")


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _hand():
    g = json.load(open(GOLD))
    ps = g["page_size"]
    pt = np.array(g["page_table"], np.int32)
    seqs = O.Seqs(ctx_len=np.array([4]), q_seq_start=np.array([0, 4]), page_table=pt, page_size=ps)
    k_log = np.array(g["kI_logical"], np.float64)
    phys = np.zeros_like(k_log)
    for s in range(4):
        phys[pt[0, s // ps] * ps + s % ps] = k_log[s]
    return g, seqs, phys


def test_hand_example_bf16():
    g, seqs, phys = _hand()
    got = O.index_scores(seqs, _bf16_bits(g["qI"]), np.array(g["w"]), _bf16_bits(phys))
    for t, row in enumerate(g["scores"]):
        assert np.array_equal(got[t], np.array(row, np.float64)), (t, got[t], row)
    topk = O.topk_rows(got, g["topk_K"])
    assert topk.tolist() == g["topk"]


def test_hand_example_fp8_cache():
    g, seqs, _ = _hand()
    ps, pt = g["page_size"], np.array(g["page_table"])
    sc_log = np.array(g["fp8_variant"]["kI_scale_logical"], np.float64)
    cv_log = np.array(g["fp8_variant"]["kI_codes_value_logical"], np.float64)
    codes = np.zeros((4, 2), np.uint8)
    scale = np.zeros(4)
    for s in range(4):
        r = pt[0, s // ps] * ps + s % ps
        codes[r] = O.e4m3_encode(cv_log[s])
        scale[r] = sc_log[s]
    assert np.array_equal(O.e4m3_decode(codes[[pt[0, s // ps] * ps + s % ps for s in range(4)]]) * sc_log[:, None],
                          np.array(g["kI_logical"], np.float64))
    got = O.index_scores(seqs, _bf16_bits(g["qI"]), np.array(g["w"]), codes, scale)
    for t, row in enumerate(g["scores"]):
        assert np.array_equal(got[t], np.array(row, np.float64)), (t, got[t], row)


def _random_case(rng, fp8, B=3, H=4, d=8, ps=4):
    ctx = rng.integers(5, 23, B)
    q_len = np.minimum(ctx, rng.integers(1, 6, B))
    pages = (ctx + ps - 1) // ps
    perm = rng.permutation(pages.sum() + 3)
    pt = np.full((B, pages.max()), -1, np.int32)
    k = 0
    for b in range(B):
        pt[b, : pages[b]] = perm[k: k + pages[b]]
        k += pages[b]
    R = (pages.sum() + 3) * ps
    qs = np.concatenate([[0], np.cumsum(q_len)])
    T = qs[-1]
    seqs = O.Seqs(ctx_len=ctx, q_seq_start=qs, page_table=pt, page_size=ps)
    qI = _bf16_bits(rng.standard_normal((T, H, d)))
    w = rng.standard_normal((T, H)) / 8
    if fp8:
        kI = rng.integers(0, 256, (R, d)).astype(np.uint8)
        kI[(kI & 0x7F) == 0x7F] = 0                 # no NaN codes
        scale = rng.uniform(0.01, 2.0, R)
    else:
        kI = _bf16_bits(rng.standard_normal((R, d)))
        scale = None
    return seqs, qI, w, kI, scale, perm, pages


def test_page_permutation_invariance():
    rng = np.random.default_rng(2)
    for fp8 in (False, True):
        seqs, qI, w, kI, scale, _, _ = _random_case(rng, fp8)
        base = O.index_scores(seqs, qI, w, kI, scale)
        # move every page to a new physical slot
        ps = seqs.page_size
        npages = kI.shape[0] // ps
        new_of_old = rng.permutation(npages)
        kI2 = np.empty_like(kI)
        for old in range(npages):
            kI2[new_of_old[old] * ps:(new_of_old[old] + 1) * ps] = kI[old * ps:(old + 1) * ps]
        sc2 = None
        if scale is not None:
            sc2 = np.empty_like(scale)
            for old in range(npages):
                sc2[new_of_old[old] * ps:(new_of_old[old] + 1) * ps] = scale[old * ps:(old + 1) * ps]
        pt2 = np.where(seqs.page_table >= 0, new_of_old[np.maximum(seqs.page_table, 0)], -1)
        seqs2 = O.Seqs(seqs.ctx_len, seqs.q_seq_start, pt2.astype(np.int32), ps)
        moved = O.index_scores(seqs2, qI, w, kI2, sc2)
        for a, b in zip(base, moved):
            assert np.array_equal(a, b)


def test_scaling_laws_and_causality():
    rng = np.random.default_rng(3)
    seqs, qI, w, kI, scale, _, _ = _random_case(rng, True)
    base = O.index_scores(seqs, qI, w, kI, scale)
    # linear in w, linear in the per-row key scale
    twice = O.index_scores(seqs, qI, 2 * w, kI, scale)
    for a, b in zip(base, twice):
        assert np.allclose(b, 2 * a, rtol=1e-15, atol=0)
    sc3 = O.index_scores(seqs, qI, w, kI, 3 * scale)
    for a, b in zip(base, sc3):
        assert np.allclose(b, 3 * a, rtol=1e-14, atol=0)
    # row length = position + 1 (the token itself is a candidate)
    for t, row in enumerate(base):
        b, pos = seqs.token_seq_pos(t)
        assert row.shape == (pos + 1,)
        assert pos == seqs.ctx_len[b] - (seqs.q_seq_start[b + 1] - seqs.q_seq_start[b]) + t - seqs.q_seq_start[b]
    # the ReLU: with all-negative head weights, no score can be positive
    neg = O.index_scores(seqs, qI, -np.abs(w), kI, scale)
    assert all(np.all(r <= 0) for r in neg)


def test_single_head_single_dim_closed_form():
    rng = np.random.default_rng(4)
    seqs = O.Seqs(ctx_len=np.array([6]), q_seq_start=np.array([0, 6]),
                  page_table=np.array([[1, 0, 2]], np.int32), page_size=2)
    qv = rng.integers(-4, 5, 6).astype(np.float64)
    kv = rng.integers(-4, 5, 6).astype(np.float64)
    wv = rng.integers(-3, 4, 6).astype(np.float64)
    kphys = np.zeros(6)
    for s in range(6):
        kphys[[1, 0, 2][s // 2] * 2 + s % 2] = kv[s]
    got = O.index_scores(seqs, _bf16_bits(qv.reshape(6, 1, 1)), wv.reshape(6, 1),
                         _bf16_bits(kphys.reshape(6, 1)))
    for t in range(6):
        want = [wv[t] * max(0.0, qv[t] * kv[s]) for s in range(t + 1)]
        assert got[t].tolist() == want
