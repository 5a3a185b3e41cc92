"""The Python binding refuses tensors the kernels would misread before any C
call: wrong device, dtype, shape, stride or pool size.  CPU only -- every
refusal here happens before the library is entered."""
import pytest
import torch

import sparse_indexed_attention_b200 as dsa

CPU = torch.device("cpu")


def test_need_accepts_a_matching_tensor():
    dsa._need(torch.zeros(3, 64, dtype=torch.float32), "w", dsa._F32T, (3, 64), CPU)
    dsa._need(torch.zeros(128, 128, dtype=torch.uint8), "kI", dsa._FP8T, (None, 128), CPU, 128)
    dsa._need(torch.zeros(128, 128, dtype=torch.float8_e4m3fn), "kI", dsa._FP8T, (None, 128), CPU, 64)


@pytest.mark.parametrize("bad, err, what", [
    (torch.zeros(3, 64, dtype=torch.float64), TypeError, "dtype"),
    (torch.zeros(3, 65, dtype=torch.float32), ValueError, "shape"),
    (torch.zeros(3, 64, 1, dtype=torch.float32), ValueError, "shape"),
    (torch.zeros(64, 3, dtype=torch.float32).t(), ValueError, "contiguous"),
    ([0.0] * 64, TypeError, "torch.Tensor"),
])
def test_need_refuses(bad, err, what):
    with pytest.raises(err, match=what):
        dsa._need(bad, "w", dsa._F32T, (3, 64), CPU)


def test_need_refuses_a_short_pool_and_another_device():
    with pytest.raises(ValueError, match="at least 128"):
        dsa._need(torch.zeros(127, 576, dtype=torch.bfloat16), "kv", dsa._BF16T, (None, 576), CPU, 128)
    with pytest.raises(ValueError, match="expected meta"):
        dsa._need(torch.zeros(4, dtype=torch.int32), "row_len", dsa._I32T, (4,), torch.device("meta"))


def test_entry_points_want_cuda_tensors():
    T, K = 2, 16
    seqs = dsa.Seqs(torch.tensor([0, 1, 2], dtype=torch.int32), torch.tensor([5, 7], dtype=torch.int32),
                    torch.zeros(2, 1, dtype=torch.int32), 2, 7, T)
    qI = torch.zeros(T, 64, 128, dtype=torch.bfloat16)
    w = torch.zeros(T, 64)
    kI = torch.zeros(128, 128, dtype=torch.bfloat16)
    q = torch.zeros(T, 16, 576, dtype=torch.bfloat16)
    kv = torch.zeros(128, 576, dtype=torch.bfloat16)
    idx = torch.zeros(T, K, dtype=torch.int32)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_quantize_index_query(qI, w)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_index_scores(seqs, qI, w, kI)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_topk(torch.zeros(T, 8), torch.full((T,), 8, dtype=torch.int32), K)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_sparse_mla_fwd(seqs, q, kv, idx, 0.1)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_sparse_mla_fwd_noalloc(seqs, q, kv, idx, 0.1)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_index_topk_attn(seqs, qI, w, kI, None, q, kv, K, 0.1)


def test_index_cache_format_follows_the_scale_dtype(monkeypatch):
    """No scale: bf16 cache; fp32 [R]: E4M3 with a row scale; uint8 [R, 4]:
    MXFP8 with E8M0 group scales.  Each form is checked against its own shape."""
    assert dsa._ki_dtype(None) == dsa.DSA_KI_BF16
    assert dsa._ki_dtype(torch.ones(128)) == dsa.DSA_KI_FP8_E4M3
    assert dsa._ki_dtype(torch.full((128, 4), 127, dtype=torch.uint8)) == dsa.DSA_KI_MXFP8
    seqs = dsa.Seqs(torch.tensor([0, 1], dtype=torch.int32), torch.tensor([5], dtype=torch.int32),
                    torch.zeros(1, 1, dtype=torch.int32), 1, 5, 1)
    qI, w = torch.zeros(1, 64, 128, dtype=torch.bfloat16), torch.zeros(1, 64)
    kI = torch.zeros(64, 128, dtype=torch.uint8)
    with pytest.raises(TypeError, match="CUDA"):
        dsa.dsa_quantize_index_query_mx(qI)
    monkeypatch.setattr(dsa, "_cuda_device", lambda t, name: t.device)  # the shape rules, on CPU tensors
    dsa._need_index_inputs(seqs, qI, w, kI, torch.full((64, 4), 127, dtype=torch.uint8))
    with pytest.raises(ValueError, match="shape"):
        dsa._need_index_inputs(seqs, qI, w, kI, torch.full((64, 2), 127, dtype=torch.uint8))
    with pytest.raises(ValueError, match="at least 64"):
        dsa._need_index_inputs(seqs, qI, w, kI, torch.full((63, 4), 127, dtype=torch.uint8))


def test_latent_cache_format_follows_kv_scale(monkeypatch):
    """kv_scale absent: a bf16 pool [R, 576]; present: E4M3 codes [R, 576] with
    uint8 scale bytes [R, 8], each checked for shape and pool size."""
    monkeypatch.setattr(dsa, "_cuda_device", lambda t, name: t.device)
    seqs = dsa.Seqs(torch.tensor([0, 1], dtype=torch.int32), torch.tensor([5], dtype=torch.int32),
                    torch.zeros(1, 1, dtype=torch.int32), 1, 5, 1)
    q = torch.zeros(1, 16, 576, dtype=torch.bfloat16)
    out = torch.zeros(1, 16, 512, dtype=torch.bfloat16)
    codes, scales = torch.zeros(64, 576, dtype=torch.uint8), torch.full((64, 8), 127, dtype=torch.uint8)
    dsa._need_attn_inputs(seqs, q, torch.zeros(64, 576, dtype=torch.bfloat16), out, None)
    dsa._need_attn_inputs(seqs, q, codes, out, None, scales)
    with pytest.raises(TypeError, match="dtype"):
        dsa._need_attn_inputs(seqs, q, codes, out, None)              # codes without their scales
    with pytest.raises(ValueError, match="shape"):
        dsa._need_attn_inputs(seqs, q, codes, out, None, scales[:, :5].contiguous())
    with pytest.raises(ValueError, match="at least 64"):
        dsa._need_attn_inputs(seqs, q, codes, out, None, scales[:63])
