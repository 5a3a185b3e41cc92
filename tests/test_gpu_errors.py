"""Bad device-side values are skipped and reported through the error flag;
nothing faults.  Every bad value here is one the kernels bounds-check."""
import numpy as np
import pytest
import torch

from dsa_workloads import to_device
from tests.specs import SMALL, workload as make_workload

pytestmark = pytest.mark.gpu


def _ws(lib, op, seqs, K=1, H=16):
    return torch.zeros(lib.dsa_workspace_size(op, seqs, K, H), dtype=torch.uint8, device="cuda")


def test_bad_page_id_sets_flag_and_clears(lib):
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    pt = d.seqs.page_table.clone()
    pt[1, 0] = wl.num_phys_pages          # one past the pool
    pt[2, 1] = -7
    seqs = lib.Seqs(d.seqs.q_seq_start, d.seqs.ctx_len, pt, d.seqs.num_phys_pages, d.seqs.max_ctx,
                    d.seqs.num_q_tokens)
    ws = _ws(lib, lib.DSA_OP_INDEX_TOPK_ATTN, seqs, wl.spec.topk, wl.spec.heads)
    lib.dsa_index_topk_attn(seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, wl.spec.topk, wl.scale, ws=ws)
    assert lib.dsa_check_error(ws) == lib.DSA_ERR_BAD_INDEX
    assert lib.dsa_check_error(ws) == lib.DSA_OK           # the flag was cleared
    # the good table runs clean on the same workspace
    lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, wl.spec.topk, wl.scale, ws=ws)
    assert lib.dsa_check_error(ws) == lib.DSA_OK


def test_bad_indices_and_lengths(lib):
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    K = wl.spec.topk
    pos = wl.token_pos()
    idx = np.full((wl.T, K), -1, np.int32)
    idx[:, 0] = pos
    idx[0, 1] = pos[0] + 1                # a future position
    idx[1, 1] = -2
    ws = _ws(lib, lib.DSA_OP_SPARSE_MLA, d.seqs, K, wl.spec.heads)
    lib.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, torch.from_numpy(idx).cuda(), wl.scale, ws=ws)
    assert lib.dsa_check_error(ws) == lib.DSA_ERR_BAD_INDEX
    # ctx_len above max_ctx, q_len above ctx_len
    cl = d.seqs.ctx_len.clone()
    cl[0] = d.seqs.max_ctx + 1
    seqs = lib.Seqs(d.seqs.q_seq_start, cl, d.seqs.page_table, d.seqs.num_phys_pages, d.seqs.max_ctx,
                    d.seqs.num_q_tokens)
    ws2 = _ws(lib, lib.DSA_OP_INDEX_TOPK_ATTN, seqs, K, wl.spec.heads)
    lib.dsa_index_topk_attn(seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, K, wl.scale, ws=ws2)
    assert lib.dsa_check_error(ws2) == lib.DSA_ERR_BAD_INDEX
    # Top-K row longer than its leading dimension
    scores = torch.randn(4, 64, device="cuda")
    row_len = torch.tensor([10, 64, 65, 3], dtype=torch.int32, device="cuda")
    ws3 = torch.zeros(lib.dsa_workspace_size(lib.DSA_OP_TOPK, None, 8, rows=4, ld=64), dtype=torch.uint8,
                      device="cuda")
    lib.dsa_topk(scores, row_len, 8, ws=ws3)
    assert lib.dsa_check_error(ws3) == lib.DSA_ERR_BAD_INDEX


def test_host_errors_raise(lib):
    wl = make_workload(SMALL["decode_small"])
    d = to_device(wl)
    small = torch.zeros(256, dtype=torch.uint8, device="cuda")
    with pytest.raises(lib.DsaError) as e:
        lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, wl.spec.topk, wl.scale, ws=small)
    assert e.value.status == lib.DSA_ERR_WORKSPACE
    with pytest.raises(lib.DsaError):
        lib.dsa_index_topk_attn(d.seqs, d.qI, d.w, d.kI, d.kI_scale, d.q, d.kv, 4096, wl.scale)
