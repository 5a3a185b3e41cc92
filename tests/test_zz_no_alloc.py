"""dsa_sparse_mla_fwd_noalloc: sparse MLA attention for callers that cannot
allocate device memory (a plugin whose host framework owns every device
allocation, or code running where cudaMalloc is not allowed).  Instead of a
caller workspace it uses a fixed scratch array inside the library.

Its results must be those of dsa_sparse_mla_fwd on the same inputs and
match the oracle; two calls in a row check that the shared array carries no
state from one call into the next, and dsa_check_error_noalloc reads the
array's error word.  The file sorts last so that a run stopping at the first
failure has already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

import sparse_indexed_attention_b200 as dsa
from dsa_workloads import bits16, to_device
from oracle import dsa_oracle as O
from tests import parity as P
from tests.specs import SMALL, workload as make_workload


def _random_selection(wl, seed):
    rng = np.random.default_rng(seed)
    pos = wl.token_pos()
    K = wl.spec.topk
    idx = np.full((wl.T, K), -1, np.int32)
    for t in range(wl.T):
        k = int(rng.integers(1, min(K, pos[t] + 1) + 1))
        idx[t, rng.choice(K, k, replace=False)] = rng.choice(pos[t] + 1, k, replace=False)
    return torch.from_numpy(idx).cuda()


@pytest.mark.gpu
def test_noalloc_matches_workspace_entry_point_on_two_calls():
    assert torch.cuda.is_available()
    # two different batches, one call each, back to back; both use the split
    # (scratch-backed) attention path since they hold fewer than 74 tokens
    cases = [(SMALL["decode_small"], 1), (SMALL["decode_b4_8k_32k"], 2)]
    for spec, seed in cases:
        wl = make_workload(spec)
        d = to_device(wl)
        idx = _random_selection(wl, seed)
        ws = torch.zeros(dsa.dsa_workspace_size(dsa.DSA_OP_SPARSE_MLA, d.seqs, wl.spec.topk, wl.spec.heads),
                         dtype=torch.uint8, device="cuda")
        ref_out, ref_lse = dsa.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, ws=ws, out_dtype=torch.float32)
        got_out, got_lse = dsa.dsa_sparse_mla_fwd_noalloc(d.seqs, d.q, d.kv, idx, wl.scale, out_dtype=torch.float32)
        torch.cuda.synchronize()
        assert dsa.dsa_check_error(ws) == dsa.DSA_OK
        assert dsa.dsa_check_error_noalloc() == dsa.DSA_OK
        ref = ref_out.double().cpu().numpy()
        rms = float(np.sqrt(np.mean(ref * ref)))
        err = float(np.abs(got_out.double().cpu().numpy() - ref).max())
        assert err <= P.OUT_TOL * rms, f"{spec.name}: max err {err:.3e} vs rms {rms:.3e}"
        lerr = (got_lse.double() - ref_lse.double()).abs().max().item()
        assert lerr <= P.LSE_TOL
        # and the oracle on the same index lists
        tokens = np.arange(wl.T)
        o_out, o_lse = O.sparse_mla(P.oracle_seqs(wl), bits16(wl.q), bits16(wl.kv), idx.cpu().numpy(), wl.scale,
                                    tokens=tokens)
        P.assert_attention_close(got_out, got_lse, o_out, o_lse)


def test_noalloc_rejects_geometry_beyond_its_scratch():
    # host-side check, answered before any CUDA call: 5 M tokens need 40 MB of token map
    fake = 0x10000
    T = 5 * 1024 * 1024
    s = dsa.DsaSeqsC(T, T, 64, 1, 1, 64, fake, fake, fake)
    need = dsa.raw().dsa_workspace_size(dsa.DSA_OP_SPARSE_MLA, ctypes.byref(s), 16, 128)
    assert need > dsa.DSA_NOALLOC_SCRATCH_BYTES
    p = ctypes.c_void_p(fake)
    st = dsa.raw().dsa_sparse_mla_fwd_noalloc(ctypes.byref(s), p, p, p, 16, 128, ctypes.c_float(0.04), p,
                                              dsa.DSA_OUT_BF16, None, None)
    assert st == dsa.DSA_ERR_WORKSPACE
