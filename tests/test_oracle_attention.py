"""Pins of the oracle's sparse MLA: with every candidate selected it equals the
dense causal masked attention, which equals torch's scaled_dot_product_attention
in float64 (a library routine); plus closed-form special cases and invariances."""
import math

import numpy as np
import torch

from oracle import dsa_oracle as O


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def _case(rng, B=2, H=3, dqk=12, dv=8, ps=4, prefill=True):
    ctx = rng.integers(3, 15, B)
    q_len = ctx.copy() if prefill else np.minimum(ctx, rng.integers(1, 4, B))
    pages = (ctx + ps - 1) // ps
    R_pages = pages.sum() + 2
    perm = rng.permutation(R_pages)
    pt = np.full((B, pages.max()), -1, np.int32)
    k = 0
    for b in range(B):
        pt[b, : pages[b]] = perm[k: k + pages[b]]
        k += pages[b]
    qs = np.concatenate([[0], np.cumsum(q_len)])
    seqs = O.Seqs(ctx_len=ctx, q_seq_start=qs, page_table=pt, page_size=ps)
    q = _bf16_bits(rng.standard_normal((qs[-1], H, dqk)))
    kv = _bf16_bits(rng.standard_normal((R_pages * ps, dqk)))
    return seqs, q, kv


def _all_idx(seqs, K):
    idx = np.full((seqs.num_tokens, K), -1, np.int32)
    for t in range(seqs.num_tokens):
        _, pos = seqs.token_seq_pos(t)
        idx[t, : pos + 1] = np.arange(pos + 1)
    return idx


def test_sparse_with_all_candidates_equals_dense():
    rng = np.random.default_rng(7)
    for prefill in (True, False):
        seqs, q, kv = _case(rng, prefill=prefill)
        K = 16
        s_out, s_lse = O.sparse_mla(seqs, q, kv, _all_idx(seqs, K), 0.3, d_v=8)
        d_out, d_lse = O.dense_masked_mla(seqs, q, kv, 0.3, d_v=8)
        assert np.allclose(s_out, d_out, rtol=1e-12, atol=1e-12)
        assert np.allclose(s_lse, d_lse, rtol=1e-12, atol=1e-12)


def test_dense_equals_torch_sdpa_fp64():
    rng = np.random.default_rng(8)
    seqs, q, kv = _case(rng, B=1, prefill=True)
    scale = 1.0 / math.sqrt(12)
    d_out, _ = O.dense_masked_mla(seqs, q, kv, scale, d_v=8)
    ctx = int(seqs.ctx_len[0])
    rows = seqs.rows(0, np.arange(ctx))
    K = torch.from_numpy(O.bf16_to_f64(kv[rows]))            # [ctx, 12]
    Q = torch.from_numpy(O.bf16_to_f64(q))                    # [ctx, H, 12]
    ref = torch.nn.functional.scaled_dot_product_attention(
        Q.transpose(0, 1), K[None].expand(Q.shape[1], -1, -1), K[None, :, :8].expand(Q.shape[1], -1, -1),
        is_causal=True, scale=scale).transpose(0, 1)
    assert np.allclose(d_out, ref.numpy(), rtol=1e-12, atol=1e-12)


def test_zero_query_gives_mean_of_selected_values():
    rng = np.random.default_rng(9)
    seqs, q, kv = _case(rng, prefill=False)
    q = np.zeros_like(q)
    idx = _all_idx(seqs, 16)
    out, lse = O.sparse_mla(seqs, q, kv, idx, 0.5, d_v=8)
    for t in range(seqs.num_tokens):
        b, pos = seqs.token_seq_pos(t)
        vals = O.bf16_to_f64(kv[seqs.rows(b, np.arange(pos + 1))])[:, :8]
        assert np.allclose(out[t], vals.mean(0)[None], rtol=1e-13, atol=1e-13)
        assert np.allclose(lse[t], math.log(pos + 1), rtol=1e-13)


def test_identical_rows_give_that_row():
    rng = np.random.default_rng(10)
    seqs, q, kv = _case(rng, prefill=False)
    kv[:] = kv[3]
    out, _ = O.sparse_mla(seqs, q, kv, _all_idx(seqs, 16), 0.5, d_v=8)
    assert np.allclose(out, O.bf16_to_f64(kv[3])[:8][None, None], rtol=1e-13, atol=1e-13)


def test_probabilities_sum_to_one_and_lse_consistent():
    rng = np.random.default_rng(11)
    seqs, q, kv = _case(rng, prefill=False)
    idx = _all_idx(seqs, 16)
    _, lse = O.sparse_mla(seqs, q, kv, idx, 0.7, d_v=8)
    for t in range(seqs.num_tokens):
        b, pos = seqs.token_seq_pos(t)
        kk = O.bf16_to_f64(kv[seqs.rows(b, np.arange(pos + 1))])
        logits = 0.7 * (O.bf16_to_f64(q[t]) @ kk.T)
        assert np.allclose(np.exp(logits - lse[t][:, None]).sum(1), 1.0, rtol=1e-13)


def test_selection_order_and_page_permutation_invariance():
    rng = np.random.default_rng(12)
    seqs, q, kv = _case(rng, prefill=True)
    K = 5
    idx = np.full((seqs.num_tokens, K), -1, np.int32)
    for t in range(seqs.num_tokens):
        _, pos = seqs.token_seq_pos(t)
        pick = rng.permutation(pos + 1)[: min(K, pos + 1)]
        idx[t, : pick.size] = np.sort(pick)
    base, base_lse = O.sparse_mla(seqs, q, kv, idx, 0.4, d_v=8)
    shuf = idx.copy()
    for t in range(seqs.num_tokens):
        rng.shuffle(shuf[t])
    got, _ = O.sparse_mla(seqs, q, kv, shuf, 0.4, d_v=8)
    assert np.allclose(got, base, rtol=1e-13, atol=1e-13)
    ps = seqs.page_size
    npages = kv.shape[0] // ps
    new_of_old = rng.permutation(npages)
    kv2 = np.empty_like(kv)
    for old in range(npages):
        kv2[new_of_old[old] * ps:(new_of_old[old] + 1) * ps] = kv[old * ps:(old + 1) * ps]
    pt2 = np.where(seqs.page_table >= 0, new_of_old[np.maximum(seqs.page_table, 0)], -1).astype(np.int32)
    got2, lse2 = O.sparse_mla(O.Seqs(seqs.ctx_len, seqs.q_seq_start, pt2, ps), q, kv2, idx, 0.4, d_v=8)
    assert np.array_equal(got2, base) and np.array_equal(lse2, base_lse)


def test_invalid_selection_rejected():
    rng = np.random.default_rng(13)
    seqs, q, kv = _case(rng, prefill=False)
    idx = np.full((seqs.num_tokens, 4), -1, np.int32)
    for t in range(seqs.num_tokens):
        _, pos = seqs.token_seq_pos(t)
        idx[t, 0] = pos + 1                      # beyond the causal boundary
    try:
        O.sparse_mla(seqs, q, kv, idx, 0.4, d_v=8)
    except ValueError:
        return
    raise AssertionError("future position accepted")
