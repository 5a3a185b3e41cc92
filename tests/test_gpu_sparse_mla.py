"""dsa_sparse_mla_fwd against the oracle on the oracle's own index sets."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from dsa_workloads import bits16, to_device
from tests import parity as P
from tests.specs import FULL, SMALL, workload as make_workload

pytestmark = pytest.mark.gpu


def _check(lib, wl, idx_np, tokens):
    d = to_device(wl)
    idx = torch.from_numpy(idx_np).cuda()
    ref_out, ref_lse = O.sparse_mla(P.oracle_seqs(wl), bits16(wl.q), P.kv_host(wl), idx_np, wl.scale,
                                    tokens=tokens)
    sel = torch.from_numpy(np.asarray(tokens)).cuda()
    for dt in (torch.float32, torch.bfloat16):
        out, lse = lib.dsa_sparse_mla_fwd(d.seqs, d.q, d.kv, idx, wl.scale, out_dtype=dt, kv_scale=d.kv_scale)
        P.assert_attention_close(out[sel], lse[sel], ref_out, ref_lse)
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "sparse_mla")) == lib.DSA_OK


@pytest.mark.parametrize("name", list(SMALL))
def test_sparse_mla_small(lib, name):
    wl = make_workload(SMALL[name])
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 64)
    ref_rows = P.oracle_scores(wl, tokens)
    idx = P.topk_idx_for(wl, ref_rows, tokens)
    if wl.T > 1100:                      # rows outside the sample still need a valid selection
        pos = wl.token_pos()
        rest = np.setdiff1d(np.arange(wl.T), tokens)
        idx[rest, 0] = pos[rest]
    _check(lib, wl, idx, tokens)


def test_sparse_mla_shuffled_and_sparse_padding(lib):
    wl = make_workload(SMALL["decode_small"])
    rng = np.random.default_rng(4)
    pos = wl.token_pos()
    K = wl.spec.topk
    idx = np.full((wl.T, K), -1, np.int32)
    for t in range(wl.T):
        k = int(rng.integers(1, min(K, pos[t] + 1) + 1))
        sel = rng.choice(pos[t] + 1, k, replace=False)
        slots = rng.choice(K, k, replace=False)      # -1 holes anywhere, any order
        idx[t, slots] = sel
    _check(lib, wl, idx, np.arange(wl.T))


def test_sparse_mla_full_decode_128k(lib):
    wl = make_workload(FULL["decode_b8_128k"])
    tokens = np.arange(wl.T)
    idx = P.topk_idx_for(wl, P.oracle_scores(wl, tokens), tokens)
    _check(lib, wl, idx, tokens)
