"""The MXFP8 index cache (E4M3 + one E8M0 scale per 32 elements) end to end
on the GPU: the query quantizer bit-exact against the oracle, the block-scaled
indexer's scores within the indexer tolerance, and the whole path (both Top-K
modes) against the oracle's selection and attention."""
import dataclasses

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O
from dsa_workloads import bits16, to_device
from tests import parity as P
from tests.specs import FULL, SMALL, workload as make_workload
from tests.test_gpu_fused import _fused_check

pytestmark = pytest.mark.gpu

MX_SMALL = {n: SMALL[n].scaled(name=n + "_mx", ki_mx=True)
            for n in ("decode_small", "prefill_fp8_700", "chunked_small", "pool_b2_128k")}


def test_quantize_index_query_mx_bit_exact(lib):
    rng = np.random.default_rng(5)
    T = 29
    # every group of 32 its own magnitude, so the four scales of a row differ
    x = rng.standard_normal((T, 64, 128)) * np.exp2(rng.integers(-60, 60, (T, 64, 4)).repeat(32, axis=2))
    x[0, 0] = 0.0                                       # zero groups -> scale byte 127
    x[0, 1, :32] = 0.0
    x[0, 1, 32:36] = [448.0, -448.0, 1.0, 0.5]          # a group whose top value sits exactly at 448 * 2^0
    x[0, 1, 36:64] = 0.0
    x[0, 2, :] = rng.standard_normal(128) * 2.0 ** -130  # bf16 subnormals: the exponent clamps at -127
    x[1, 0, :32] = 3.9 * 2.0 ** np.arange(-16, 16)      # one group spanning 32 binades: small values underflow
    qI = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16)
    codes, scales = lib.dsa_quantize_index_query_mx(qI.cuda())
    ref_codes, ref_scales = O.mxfp8_quantize(O.bf16_to_f64(bits16(qI)))
    fold = lambda c: np.where((c & 0x7F) == 0, 0, c)  # noqa: E731  (+0 and -0 are one value)
    assert np.array_equal(scales.cpu().numpy(), ref_scales)
    assert np.array_equal(fold(codes.cpu().numpy()), fold(ref_codes))


@pytest.mark.parametrize("name", list(MX_SMALL))
def test_index_scores_mx_small(lib, name):
    wl = make_workload(MX_SMALL[name])
    d = to_device(wl)
    assert d.kI_scale.dtype == torch.uint8
    scores = lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale)
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 64)
    P.assert_scores_close(P.device_rows(scores, wl, tokens), P.oracle_scores(wl, tokens), tokens)
    assert lib.dsa_check_error(lib.workspace(0, "cuda", "index_scores")) == lib.DSA_OK


def test_index_scores_mx_full_decode(lib):
    wl = make_workload(FULL["decode_b8_128k"].scaled(name="decode_b8_128k_mx", ki_mx=True))
    d = to_device(wl)
    scores = lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale)
    tokens = np.arange(wl.T)
    P.assert_scores_close(P.device_rows(scores, wl, tokens), P.oracle_scores(wl, tokens), tokens)


@pytest.mark.parametrize("name", list(MX_SMALL))
def test_whole_path_mx(lib, name):
    wl = make_workload(MX_SMALL[name])
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 48)
    _fused_check(lib, wl, tokens, out_dtype=torch.float32)
    if wl.T == wl.spec.batch:                            # decode: the selection inside the indexer too
        _fused_check(lib, wl, tokens, out_dtype=torch.float32, select_in_indexer=True)


def test_mx_scales_are_applied(lib):
    """Doubling one key group's scale (E8M0 byte + 1) must change exactly the
    scores that group contributes to: a check that the kernel reads each
    group's byte and not a neighbour's."""
    wl = make_workload(MX_SMALL["decode_small"])
    d = to_device(wl)
    base = lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, d.kI_scale).clone()
    sc = d.kI_scale.clone()
    sc[:, 2] += 1
    moved = lib.dsa_index_scores(d.seqs, d.qI, d.w, d.kI, sc)
    wl2 = dataclasses.replace(wl, kI_scale=sc.cpu())
    tokens = np.arange(wl.T)
    P.assert_scores_close(P.device_rows(moved, wl2, tokens), P.oracle_scores(wl2, tokens), tokens)
    assert not torch.equal(base, moved)
