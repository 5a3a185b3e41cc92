"""Every compute entry point's host path returns promptly.  On a machine
without a GPU each call runs its argument checks, workspace carve-up and
dispatch on the host and then fails at its first CUDA call with
DSA_ERR_CUDA; a call that loops or blocks on the host would time out here.
The buffers are host memory, so the test never runs where a GPU is present."""
import pytest
import torch

import sparse_indexed_attention_b200 as dsa
from dsa_workloads import CONFIGS, make_workload

pytestmark = [pytest.mark.timeout(60),
              pytest.mark.skipif(torch.cuda.is_available(), reason="host buffers must not reach a GPU launch")]


def _aligned(t):
    n = t.numel() * t.element_size()
    buf = torch.empty(n + 256, dtype=torch.uint8)
    off = (-buf.data_ptr()) % 256
    out = buf[off:off + n].view(t.dtype).view(t.shape)
    out.copy_(t)
    return out


@pytest.fixture
def host_binding(monkeypatch):
    monkeypatch.setattr(dsa, "_cuda_device", lambda t, name: t.device)
    monkeypatch.setattr(dsa, "_stream", lambda dev: None)
    monkeypatch.setattr(dsa, "workspace", lambda n, dev, key=None: _aligned(torch.zeros(max(n, 256), dtype=torch.uint8)))
    return dsa


def _inputs(spec):
    wl = make_workload(spec)
    seqs = dsa.Seqs(*(_aligned(torch.from_numpy(x)) for x in (wl.q_seq_start, wl.ctx_len, wl.page_table)),
                    wl.num_phys_pages, int(wl.ctx_len.max()), wl.T)
    ks = None if wl.kI_scale is None else _aligned(wl.kI_scale)
    vs = None if wl.kv_scale is None else _aligned(wl.kv_scale)
    return wl, seqs, _aligned(wl.qI), _aligned(wl.w), _aligned(wl.kI), ks, _aligned(wl.q), _aligned(wl.kv), vs


SPECS = {
    "bf16_prefill": CONFIGS["tiny_prefill_1k"],
    "fp8_prefill": CONFIGS["long_prefill_32k"].scaled(ctx=(2048, 2048)),
    "mx_prefill": CONFIGS["long_prefill_32k"].scaled(ctx=(2048, 2048), ki_mx=True),
    "fp8_decode": CONFIGS["decode_b64_8k_32k"].scaled(batch=3),
    "mx_decode": CONFIGS["decode_b64_8k_32k"].scaled(batch=3, ki_mx=True),
    "kv8_decode": CONFIGS["decode_b64_8k_32k"].scaled(batch=3, kv_fp8=True),
}


@pytest.mark.parametrize("name", list(SPECS))
def test_entry_points_return_without_a_gpu(host_binding, name):
    wl, seqs, qI, w, kI, ks, q, kv, vs = _inputs(SPECS[name])
    K = wl.spec.topk
    scores = _aligned(torch.zeros((wl.T, (wl.max_ctx + 3) // 4 * 4), dtype=torch.float32))
    out = _aligned(torch.zeros((wl.T, wl.spec.heads, 512), dtype=torch.bfloat16))
    lse = _aligned(torch.zeros((wl.T, wl.spec.heads), dtype=torch.float32))
    idx = _aligned(torch.zeros((wl.T, K), dtype=torch.int32))
    codes = _aligned(torch.zeros((wl.T, 64, 128), dtype=torch.float8_e4m3fn))
    w_scaled = _aligned(torch.zeros((wl.T, 64), dtype=torch.float32))
    q_sf = _aligned(torch.zeros((wl.T, 64, 4), dtype=torch.uint8))
    row_len = _aligned(torch.full((wl.T,), scores.shape[1], dtype=torch.int32))
    calls = [
        lambda: dsa.dsa_index_scores(seqs, qI, w, kI, ks, scores=scores),
        lambda: dsa.dsa_sparse_mla_fwd(seqs, q, kv, idx, wl.scale, out=out, lse=lse, kv_scale=vs),
        lambda: dsa.dsa_index_topk_attn(seqs, qI, w, kI, ks, q, kv, K, wl.scale, out=out, lse=lse, kv_scale=vs),
        lambda: dsa.dsa_index_topk_attn(seqs, qI, w, kI, ks, q, kv, K, wl.scale, out=out, lse=lse,
                                        select_in_indexer=True, kv_scale=vs),
        lambda: dsa.dsa_quantize_index_query(qI, w, codes=codes, w_scaled=w_scaled),
        lambda: dsa.dsa_quantize_index_query_mx(qI, codes=codes, scales=q_sf),
        lambda: dsa.dsa_topk(scores, row_len, K, idx=idx),
    ]
    if vs is None:  # the allocation-free attention reads the bf16 latent pool only
        calls.append(lambda: dsa.dsa_sparse_mla_fwd_noalloc(seqs, q, kv, idx, wl.scale, out=out, lse=lse))
    for call in calls:
        with pytest.raises(dsa.DsaError, match="DSA_ERR_CUDA"):
            call()
