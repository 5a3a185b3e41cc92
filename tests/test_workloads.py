"""The seeded generator: deterministic, valid page tables, stated shapes."""
import numpy as np
import torch

from dsa_workloads import CONFIGS, make_workload

SMALL = {
    "prefill": CONFIGS["tiny_prefill_1k"].scaled(ctx=(300, 300), topk=64),
    "decode": CONFIGS["decode_b64_8k_32k"].scaled(batch=5, ctx=(100, 700), topk=128, planted=8),
    "chunked": CONFIGS["chunked_prefill_16"].scaled(batch=3, prefix=(0, 500), chunk=(10, 90), topk=64),
    "pool": CONFIGS["decode_b8_128k"].scaled(batch=2, ctx=(1000, 1000), pool_tokens=64 * 100, topk=128),
}


def test_deterministic_and_valid():
    for name, spec in SMALL.items():
        a, b = make_workload(spec), make_workload(spec)
        for f in ("qI", "w", "kI", "q", "kv"):
            assert torch.equal(getattr(a, f), getattr(b, f)), (name, f)
        assert np.array_equal(a.page_table, b.page_table)
        B = spec.batch
        assert a.ctx_len.shape == (B,) and a.q_seq_start.shape == (B + 1,)
        used = a.page_table[a.page_table >= 0]
        assert used.size == np.unique(used).size                   # no page shared
        assert used.max() < a.num_phys_pages
        for bb in range(B):
            need = (a.ctx_len[bb] + 63) // 64
            assert np.all(a.page_table[bb, :need] >= 0) and np.all(a.page_table[bb, need:] < 0)
        T = a.T
        assert a.qI.shape == (T, 64, 128) and a.qI.dtype == torch.bfloat16
        assert a.q.shape == (T, spec.heads, 576) and a.kv.shape == (a.num_phys_pages * 64, 576)
        if spec.ki_fp8:
            assert a.kI.dtype == torch.uint8 and a.kI_scale.shape == (a.num_phys_pages * 64,)
            assert not torch.any((a.kI & 0x7F) == 0x7F)            # no NaN codes
        pos = a.token_pos()
        for bb in range(B):
            seg = pos[a.q_seq_start[bb]:a.q_seq_start[bb + 1]]
            assert seg[-1] == a.ctx_len[bb] - 1 and np.all(np.diff(seg) == 1) and seg[0] >= 0


def test_modes():
    d = make_workload(SMALL["decode"])
    assert np.all(d.q_len == 1)
    assert all(p.size == 8 for p in d.planted)
    c = make_workload(SMALL["chunked"])
    assert np.all(c.q_len <= c.ctx_len) and np.all(c.q_len >= 10)
    p = make_workload(SMALL["pool"])
    assert p.num_phys_pages == 100


def test_mx_cache_rows_are_mxfp8_encodings():
    """Every MXFP8 cache row is a fixed point of the format: its decoded values
    quantize back to the same codes and scales (each block's largest code lies
    in E4M3's top binade, as the shared-exponent rule puts it)."""
    from oracle import dsa_oracle as O
    spec = CONFIGS["decode_b64_8k_32k"].scaled(batch=2, ctx=(300, 700), ki_mx=True, planted=8)
    wl = make_workload(spec)
    codes, sc = wl.kI.numpy(), wl.kI_scale.numpy()
    assert codes.dtype == np.uint8 and sc.shape == (codes.shape[0], 4)
    c2, s2 = O.mxfp8_quantize(O.mxfp8_dequantize(codes, sc))
    assert np.array_equal(c2, codes) and np.array_equal(s2, sc)
    used = np.abs(O.mxfp8_dequantize(codes, sc)).reshape(-1, 4, 32).max(-1) > 0
    assert used.mean() > 0.5


def test_fp8_kv_cache_rows_follow_the_tile_scale_rule():
    """Each tile of the FP8 latent cache is stored with the tightest
    power-of-two scale: its largest code magnitude lies in [224, 448] (amax in
    (224, 448] x 2^e before rounding); zero tiles carry scale byte 127, the
    padding bytes are zero, unused pool rows decode to zero."""
    from oracle import dsa_oracle as O
    spec = CONFIGS["decode_b64_8k_32k"].scaled(batch=2, ctx=(300, 700), kv_fp8=True, planted=8)
    wl = make_workload(spec)
    codes, sc = wl.kv.numpy(), wl.kv_scale.numpy()
    assert codes.dtype == np.uint8 and sc.shape == (codes.shape[0], 8) and np.all(sc[:, 5:] == 0)
    mag = np.abs(O.e4m3_decode_fast(codes))
    for j, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 384), (384, 512), (512, 576)]):
        top = mag[:, lo:hi].max(axis=1)
        nz = top > 0
        assert np.all((top[nz] >= 224.0) & (top[nz] <= 448.0))
        assert np.all(sc[~nz, j] == 127)
    used = np.abs(O.kv_fp8_dequantize(codes, sc)).max(axis=1) > 0
    assert 0.5 < used.mean() <= 1.0
