"""dsa_index_topk_attn end to end: the selection criterion against the oracle's
scores, and attention parity on every row whose index set equals the
oracle's (the oracle never consumes a GPU result)."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from dsa_workloads import bits16, to_device
from tests import parity as P
from tests.specs import FULL, SMALL, workload as make_workload

pytestmark = pytest.mark.gpu


def _fused_check(lib, wl, tokens, min_agree=0.9, out_dtype=torch.bfloat16, select_in_indexer=False):
    d = to_device(wl)
    K = wl.spec.topk
    idx_out = torch.empty((wl.T, K), dtype=torch.int32, device="cuda")
    out, lse = lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                       idx_out=idx_out, out_dtype=out_dtype, select_in_indexer=select_in_indexer,
                                       kv_scale=d.kv_scale)
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "index_topk_attn")) == lib.DSA_OK
    gidx = idx_out.cpu().numpy()
    ref_rows = P.oracle_scores(wl, tokens)
    agree = []
    for t, r in zip(tokens, ref_rows):
        bad = P.selection_violations(gidx[t], r, K)
        assert not bad, f"token {t}: selection differs beyond near-ties: {bad[:8]}"
        valid = gidx[t][gidx[t] >= 0]
        assert np.all(np.diff(valid) > 0)                       # ascending, no duplicates
        if np.array_equal(gidx[t], O.topk_select(r, K)):
            agree.append(t)
    assert len(agree) >= min_agree * len(tokens), f"{len(agree)}/{len(tokens)} rows with identical sets"
    ref_idx = P.topk_idx_for(wl, [ref_rows[list(tokens).index(t)] for t in agree], agree)
    ref_out, ref_lse = O.sparse_mla(P.oracle_seqs(wl), bits16(wl.q), P.kv_host(wl), ref_idx, wl.scale,
                                    tokens=agree)
    sel = torch.from_numpy(np.asarray(agree)).cuda()
    P.assert_attention_close(out[sel], lse[sel], ref_out, ref_lse)


# DSA_SELECT_IN_INDEXER changes decode batches only (one query token per sequence)
DECODE = {"decode_small", "decode_b4_8k_32k", "pool_b2_128k", "decode_b8_128k", "decode_b64_8k_32k"}


@pytest.mark.parametrize("name", list(SMALL))
def test_fused_small(lib, name):
    wl = make_workload(SMALL[name])
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 64)
    _fused_check(lib, wl, tokens, out_dtype=torch.float32)
    _fused_check(lib, wl, tokens, out_dtype=torch.bfloat16)
    if name in DECODE:
        _fused_check(lib, wl, tokens, out_dtype=torch.float32, select_in_indexer=True)


@pytest.mark.parametrize("name", ["decode_b8_128k", "decode_b64_8k_32k", "chunked_prefill_16", "long_prefill_32k"])
def test_fused_full_size(lib, name):
    wl = make_workload(FULL[name])
    tokens = np.arange(wl.T) if wl.T <= 8 else P.sample_tokens(wl, 24)
    _fused_check(lib, wl, tokens)
    if name in DECODE:
        _fused_check(lib, wl, tokens, select_in_indexer=True)


def test_fused_workspace_reused_across_geometries(lib):
    """One workspace, sized for the largest call, serves calls of different
    shapes back to back; state a call leaves behind must not leak into the next."""
    specs = [SMALL["pool_b2_128k"], SMALL["decode_b4_8k_32k"], SMALL["decode_small"], SMALL["pool_b2_128k"]]
    wls = [make_workload(s) for s in specs]
    devs = [to_device(w) for w in wls]
    need = max(lib.dsa_workspace_size(lib.DSA_OP_INDEX_TOPK_ATTN, d.seqs, w.spec.topk, w.spec.heads)
               for w, d in zip(wls, devs))
    ws = torch.zeros(need, dtype=torch.uint8, device="cuda")
    ws[256:].fill_(0xA5)  # everything but the error word starts dirty
    for wl, d in zip(wls, devs):
        K = wl.spec.topk
        idx_out = torch.empty((wl.T, K), dtype=torch.int32, device="cuda")
        lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, idx_out=idx_out,
                                ws=ws)
        assert lib.dsa_check_error(ws) == lib.DSA_OK
        gidx = idx_out.cpu().numpy()
        tokens = np.arange(wl.T)
        for t, r in zip(tokens, P.oracle_scores(wl, tokens)):
            assert not P.selection_violations(gidx[t], r, K)


def test_fused_tied_rows_take_the_lowest_positions(lib):
    """A decode row whose scores all tie (its index cache is zero, so every
    score is 0) must select exactly positions 0 .. K-1.  With the selection
    inside the indexer, that row keeps 131072 candidates -- more than a row's
    candidate list holds -- and takes the row-histogram path, while the other
    row of the same call takes the candidate-list path.  Both modes must
    match the oracle."""
    import dataclasses
    wl = make_workload(SMALL["pool_b2_128k"])
    kI = wl.kI.clone()
    pages = wl.page_table[0][wl.page_table[0] >= 0].astype(np.int64)
    rows = torch.from_numpy((pages[:, None] * 64 + np.arange(64)[None, :]).reshape(-1))
    kI[rows] = 0                                                # E4M3 code 0 = 0.0
    wl = dataclasses.replace(wl, kI=kI)
    K = wl.spec.topk
    tokens = np.arange(wl.T)
    d = to_device(wl)
    for sel in (True, False):
        _fused_check(lib, wl, tokens, min_agree=1.0, select_in_indexer=sel)
        idx_out = torch.empty((wl.T, K), dtype=torch.int32, device="cuda")
        lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, idx_out=idx_out,
                                select_in_indexer=sel)
        assert np.array_equal(idx_out[0].cpu().numpy(), np.arange(K))


@pytest.mark.parametrize("select_in_indexer", [False, True])
def test_fused_attention_waits_for_q_ready(lib, select_in_indexer):
    """dsa_index_topk_attn_ex: the attention query arrives on another stream,
    late (a spin kernel runs first); the attention launch waits on its event,
    so the result equals the call made with q already in place."""
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    K = wl.spec.topk
    ref_out, ref_lse = lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                               out_dtype=torch.float32, select_in_indexer=select_in_indexer)
    ref_out, ref_lse = ref_out.clone(), ref_lse.clone()
    q_final = d.q.clone()
    d.q.zero_()
    torch.cuda.synchronize()
    side = torch.cuda.Stream()
    ev = torch.cuda.Event()
    with torch.cuda.stream(side):
        torch.cuda._sleep(20_000_000)              # ~10 ms at 2 GHz: the indexer is long done
        d.q.copy_(q_final)
        ev.record(side)
    out, lse = lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                       out_dtype=torch.float32, q_ready=ev, select_in_indexer=select_in_indexer)
    torch.cuda.synchronize()
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "index_topk_attn")) == lib.DSA_OK
    assert not torch.equal(out[:, 0], out[:, 1])      # a zero query would give every head the same row
    assert torch.equal(out, ref_out) and torch.equal(lse, ref_lse)
