"""Pins of the oracle's FP8 latent KV cache: a hand-expanded row, the tile
boundaries (four tiles of 128 and the 64 rope dims), the tightest power-of-two
scale, exactness in bf16, the error bound, and attention over an FP8 cache equal
to attention over the same values stored as bf16."""
import json
import os

import numpy as np
import torch

from oracle import dsa_oracle as O

HAND = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "kv_fp8_hand_row.json")))


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_hand_row():
    x = np.zeros((1, 576))
    for k, v in HAND["nonzero"].items():
        x[0, int(k)] = v
    codes, scales = O.kv_fp8_quantize(x)
    assert scales[0].tolist() == HAND["scales"]
    for k, c in HAND["codes"].items():
        assert codes[0, int(k)] == c, k
    nz = set(int(k) for k in HAND["codes"])
    assert all(codes[0, i] == 0 for i in range(576) if i not in nz)
    vals = O.kv_fp8_dequantize(codes, scales)
    for k, v in HAND["values"].items():
        assert vals[0, int(k)] == v


def test_tiles_are_independent_and_bounded_where_the_pages_put_them():
    rng = np.random.default_rng(21)
    x = rng.standard_normal((40, 576))
    codes, scales = O.kv_fp8_quantize(x)
    assert np.all(scales[:, 5:] == 0)
    edges = [0, 128, 256, 384, 512, 576]
    for j in range(5):
        y = x.copy()
        y[:, edges[j]:edges[j + 1]] *= 2.0 ** 12           # one tile much larger
        c2, s2 = O.kv_fp8_quantize(y)
        others = np.r_[0:edges[j], edges[j + 1]:576]
        assert np.array_equal(c2[:, others], codes[:, others])
        assert np.array_equal(np.delete(s2[:, :5], j, axis=1), np.delete(scales[:, :5], j, axis=1))
        assert np.array_equal(c2[:, edges[j]:edges[j + 1]], codes[:, edges[j]:edges[j + 1]])
        assert np.all(s2[:, j].astype(int) == scales[:, j].astype(int) + 12)


def test_tightest_scale_no_saturation_and_error_bound():
    rng = np.random.default_rng(22)
    x = rng.standard_normal((60, 576)) * np.exp2(rng.integers(-20, 20, (60, 1)))
    codes, scales = O.kv_fp8_quantize(x)
    rec = O.kv_fp8_dequantize(codes, scales)
    for j, (lo, hi) in enumerate([(0, 128), (128, 256), (256, 384), (384, 512), (512, 576)]):
        s = O.e8m0_decode(scales[:, j])[:, None]
        amax = np.abs(x[:, lo:hi]).max(axis=1, keepdims=True)
        assert np.all(amax / s <= 448.0)                  # nothing saturates
        assert np.all(amax / s > 224.0)                   # half the scale would saturate
        err = np.abs(rec[:, lo:hi] - x[:, lo:hi])
        assert np.all(err <= np.maximum(np.abs(x[:, lo:hi]) * 2.0 ** -4, s * 2.0 ** -10))


def test_dequantized_values_are_bf16_numbers():
    rng = np.random.default_rng(23)
    codes, scales = O.kv_fp8_quantize(rng.standard_normal((30, 576)) * 7.0)
    v = O.kv_fp8_dequantize(codes, scales)
    assert np.array_equal(O.bf16_to_f64(_bf16_bits(v)), v)


def test_attention_over_fp8_cache_equals_attention_over_its_values():
    rng = np.random.default_rng(24)
    ps, H = 4, 3
    seqs = O.Seqs(ctx_len=np.array([11, 7]), q_seq_start=np.array([0, 2, 3]),
                  page_table=np.array([[2, 0, 4], [1, 3, -1]], np.int32), page_size=ps)
    R = 5 * ps
    codes, scales = O.kv_fp8_quantize(rng.standard_normal((R, 576)))
    q = _bf16_bits(rng.standard_normal((3, H, 576)))
    idx = np.full((3, 4), -1, np.int32)
    idx[0, :3] = [0, 5, 9]
    idx[1, :4] = [10, 3, 1, 7]
    idx[2, :2] = [6, 2]
    got = O.sparse_mla(seqs, q, (codes, scales), idx, 0.05)
    want = O.sparse_mla(seqs, q, _bf16_bits(O.kv_fp8_dequantize(codes, scales)), idx, 0.05)
    assert np.array_equal(got[0], want[0]) and np.array_equal(got[1], want[1])
    # the scales matter: one tile's scale doubled moves the outputs that read that row
    sc2 = scales.copy()
    sc2[seqs.rows(0, [5])[0], 4] += 1
    moved = O.sparse_mla(seqs, q, (codes, sc2), idx, 0.05)
    assert not np.array_equal(moved[0][0], got[0][0]) and np.array_equal(moved[0][2], got[0][2])
