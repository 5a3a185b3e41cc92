"""Bounded in-kernel waits.  A wait limit set far too short (1 ns) makes the
kernels' waits run out on purpose: the call must report DSA_ERR_TIMEOUT
through the workspace's error word, its CTAs must wind down by themselves
(draining only the copies and MMAs they issued), and the next call with the
default limit must run clean and match the oracle.  Nothing here faults or
hangs a GPU: the kernels give up on their own and return."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from dsa_workloads import bits16, to_device
from tests import parity as P
from tests.specs import SMALL, workload as make_workload

pytestmark = pytest.mark.gpu


def _short_limit(lib, fn):
    lib.dsa_set_wait_limit_ns(1)
    try:
        fn()
    finally:
        lib.dsa_set_wait_limit_ns(0)


def test_attention_wait_runs_out_then_next_call_is_clean(lib):
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    K, H = wl.spec.topk, wl.spec.heads
    tokens = np.arange(wl.T)
    idx_np = P.topk_idx_for(wl, P.oracle_scores(wl, tokens), tokens)
    idx = torch.from_numpy(idx_np).cuda()
    ws = torch.zeros(lib.dsa_workspace_size(lib.DSA_OP_SPARSE_MLA, d.seqs, K, H), dtype=torch.uint8, device="cuda")
    # the MMA issuer finds nothing ready while the loaders resolve the first
    # block's rows (two dependent global round trips), so its wait runs out
    _short_limit(lib, lambda: lib.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, ws=ws))
    assert lib.dsa_check_error(ws) == lib.DSA_ERR_TIMEOUT
    assert lib.dsa_check_error(ws) == lib.DSA_OK                  # reading the word clears it
    out, lse = lib.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, ws=ws, out_dtype=torch.float32)
    assert lib.dsa_check_error(ws) == lib.DSA_OK
    ref_out, ref_lse = O.sparse_mla(P.oracle_seqs(wl), bits16(wl.q), bits16(wl.kv), idx_np, wl.scale,
                                    tokens=tokens)
    P.assert_attention_close(out, lse, ref_out, ref_lse)


def test_fused_wait_runs_out_then_next_call_is_clean(lib):
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    K, H = wl.spec.topk, wl.spec.heads
    ws = torch.zeros(lib.dsa_workspace_size(lib.DSA_OP_INDEX_TOPK_ATTN, d.seqs, K, H), dtype=torch.uint8,
                     device="cuda")
    idx_out = torch.empty((wl.T, K), dtype=torch.int32, device="cuda")

    def call(**kw):
        return lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, ws=ws,
                                       idx_out=idx_out, **kw)

    _short_limit(lib, call)
    assert lib.dsa_check_error(ws) == lib.DSA_ERR_TIMEOUT
    # the selection inside the indexer waits across CTAs too: let those waits run out
    ws_f = torch.zeros(lib.dsa_workspace_size(lib.DSA_OP_INDEX_TOPK_ATTN_FUSED, d.seqs, K, H), dtype=torch.uint8,
                       device="cuda")
    _short_limit(lib, lambda: lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale,
                                                      ws=ws_f, select_in_indexer=True))
    assert lib.dsa_check_error(ws_f) == lib.DSA_ERR_TIMEOUT
    out, lse = call(out_dtype=torch.float32)
    assert lib.dsa_check_error(ws) == lib.DSA_OK
    tokens = np.arange(wl.T)
    ref_rows = P.oracle_scores(wl, tokens)
    gidx = idx_out.cpu().numpy()
    for t, r in zip(tokens, ref_rows):
        assert not P.selection_violations(gidx[t], r, K), f"token {t}"
    ref_out, ref_lse = O.sparse_mla(P.oracle_seqs(wl), bits16(wl.q), bits16(wl.kv), gidx, wl.scale, tokens=tokens)
    P.assert_attention_close(out, lse, ref_out, ref_lse)


def test_indexer_short_limit_winds_down_and_recovers(lib):
    # whether one of the indexer's waits outlasts 1 ns depends on timing, so
    # either status is accepted; what must hold is the wind-down (no fault,
    # nothing left in flight) and a clean, correct next call
    wl = make_workload(SMALL["decode_b4_8k_32k"])
    d = to_device(wl)
    ws = torch.zeros(lib.dsa_workspace_size(lib.DSA_OP_INDEX_SCORES, d.seqs, 1, 16), dtype=torch.uint8,
                     device="cuda")
    scores = torch.zeros((wl.T, (wl.max_ctx + 3) // 4 * 4), dtype=torch.float32, device="cuda")
    _short_limit(lib, lambda: lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores, ws=ws))
    assert lib.dsa_check_error(ws) in (lib.DSA_OK, lib.DSA_ERR_TIMEOUT)
    lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores, ws=ws)
    assert lib.dsa_check_error(ws) == lib.DSA_OK
    tokens = np.arange(wl.T)
    P.assert_scores_close(P.device_rows(scores, wl, tokens), P.oracle_scores(wl, tokens), tokens)
