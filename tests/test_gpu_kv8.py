"""The FP8 latent KV cache (E4M3, one power-of-two scale per 128-element tile)
on the GPU: attention on the oracle's own index sets, at reduced and full size,
and the whole path, against the oracle attending over the same cache."""
import numpy as np
import pytest
import torch

from dsa_workloads import to_device
from tests import parity as P
from tests.specs import FULL, SMALL, workload as make_workload
from tests.test_gpu_fused import _fused_check
from tests.test_gpu_sparse_mla import _check

pytestmark = pytest.mark.gpu

KV8_SMALL = {n: SMALL[n].scaled(name=n + "_kv8", kv_fp8=True)
             for n in ("decode_small", "prefill_fp8_700", "chunked_small", "tiny_prefill_1k")}


@pytest.mark.parametrize("name", list(KV8_SMALL))
def test_sparse_mla_kv8_small(lib, name):
    wl = make_workload(KV8_SMALL[name])
    assert wl.kv.dtype == torch.uint8 and wl.kv_scale is not None
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 64)
    ref_rows = P.oracle_scores(wl, tokens)
    idx = P.topk_idx_for(wl, ref_rows, tokens)
    if wl.T > 1100:                      # rows outside the sample still need a valid selection
        pos = wl.token_pos()
        rest = np.setdiff1d(np.arange(wl.T), tokens)
        idx[rest, 0] = pos[rest]
    _check(lib, wl, idx, tokens)


def test_sparse_mla_kv8_full_decode(lib):
    wl = make_workload(FULL["decode_b8_128k"].scaled(name="decode_b8_128k_kv8", kv_fp8=True))
    tokens = np.arange(wl.T)
    idx = P.topk_idx_for(wl, P.oracle_scores(wl, tokens), tokens)
    _check(lib, wl, idx, tokens)


@pytest.mark.parametrize("name", ["decode_small", "prefill_fp8_700"])
def test_whole_path_kv8(lib, name):
    wl = make_workload(KV8_SMALL[name])
    tokens = np.arange(wl.T) if wl.T <= 1100 else P.sample_tokens(wl, 48)
    _fused_check(lib, wl, tokens, out_dtype=torch.float32)
