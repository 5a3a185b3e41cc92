"""dsa_quantize_index_query (bit-exact codes) and dsa_index_scores (per-row
1e-2 x rms) against the oracle, on reduced and full-size workloads."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from dsa_workloads import bits16, to_device
from tests import parity as P
from tests.specs import FULL, SMALL, workload as make_workload

pytestmark = pytest.mark.gpu

SENTINEL = 12345.0


def test_quantize_index_query_bit_exact(lib):
    rng = np.random.default_rng(0)
    T = 37
    x = rng.standard_normal((T, 64, 128)) * np.exp2(rng.integers(-20, 20, (T, 64, 1)))
    x[0, 0] = 0.0                                      # zero row -> scale 1
    x[0, 1, :4] = [448.0, -448.0, 1.0, 0.5]            # exact boundary
    x[0, 1, 4:] = 0.0
    qI = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    w = torch.from_numpy(rng.standard_normal((T, 64)).astype(np.float32))
    codes, w_scaled = lib.dsa_quantize_index_query(qI.cuda(), w.cuda())
    ref_codes, sq = O.quantize_index_query(bits16(qI))
    got = codes.cpu().numpy()
    # +0 and -0 are one value; compare codes with zero folded
    fold = lambda c: np.where((c & 0x7F) == 0, 0, c)  # noqa: E731
    assert np.array_equal(fold(got), fold(ref_codes))
    assert np.array_equal(w_scaled.cpu().numpy().astype(np.float64), w.numpy().astype(np.float64) * sq)


@pytest.mark.parametrize("name", list(SMALL))
def test_index_scores_small(lib, name):
    wl = make_workload(SMALL[name])
    d = to_device(wl)
    ld = (wl.max_ctx + 3) // 4 * 4 + 4
    scores = torch.full((wl.T, ld), SENTINEL, dtype=torch.float32, device="cuda")
    lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale, scores=scores, ld=ld)
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 64)
    ref = P.oracle_scores(wl, tokens)
    got = P.device_rows(scores, wl, tokens)
    P.assert_scores_close(got, ref, tokens)
    host = scores.cpu().numpy()
    pos = wl.token_pos()
    for t in tokens:                                   # entries past pos untouched
        assert np.all(host[t, pos[t] + 1:] == SENTINEL)
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "index_scores")) == lib.DSA_OK


@pytest.mark.parametrize("name", ["decode_b8_128k", "decode_b64_8k_32k"])
def test_index_scores_full_decode(lib, name):
    wl = make_workload(FULL[name])
    d = to_device(wl)
    scores = lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale)
    tokens = np.arange(wl.T) if wl.T <= 8 else P.sample_tokens(wl, 12)
    P.assert_scores_close(P.device_rows(scores, wl, tokens), P.oracle_scores(wl, tokens), tokens)
