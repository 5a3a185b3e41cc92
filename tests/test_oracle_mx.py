"""Pins of the oracle's MXFP8 codec and MXFP8 indexer: a hand-expanded block,
the E8M0 scale values, the shared-exponent rule at every binade boundary, a
brute-force quantizer on random blocks, the error bound, and the indexer's
hand-expanded example in MXFP8 form."""
import json
import math
import os

import numpy as np
import torch

from oracle import dsa_oracle as O

HERE = os.path.dirname(__file__)
BLOCK = json.load(open(os.path.join(HERE, "golden", "mxfp8_hand_block.json")))
HAND = json.load(open(os.path.join(HERE, "golden", "indexer_hand_4tok.json")))


def _block(head):
    x = np.zeros(32)
    x[: len(head)] = head
    return x


def test_hand_block():
    for case in (BLOCK, BLOCK["saturation"], BLOCK["saturation_above_448"]):
        codes, sc = O.mxfp8_quantize(_block(case["x_head"]))
        n = len(case["codes_head"])
        assert codes[:n].tolist() == case["codes_head"], case
        assert np.all(codes[n:] == 0)
        assert sc.tolist() == [case["scale_code"]]
    vals = O.mxfp8_dequantize(*O.mxfp8_quantize(_block(BLOCK["x_head"])))
    assert vals[:8].tolist() == BLOCK["values_head"]


def test_e8m0_values():
    c = np.arange(256, dtype=np.uint8)
    v = O.e8m0_decode(c)
    for k in range(255):
        assert v[k] == math.ldexp(1.0, k - 127)
    assert np.isnan(v[255])


def test_shared_exponent_at_binade_edges():
    for k in range(-118, 120):
        lo = math.ldexp(1.0, k)
        assert O.mx_shared_exponent(lo) == k - 8                       # amax = 2^k
        assert O.mx_shared_exponent(np.nextafter(2 * lo, 0.0)) == k - 8  # just below 2^(k+1)
        assert O.mx_shared_exponent(1.5 * lo) == k - 8
    assert O.mx_shared_exponent(0.0) == 0
    assert O.mx_shared_exponent(math.ldexp(1.0, -140)) == -127          # clamped to E8M0's range
    assert O.mx_shared_exponent(448.0) == 0 and O.mx_shared_exponent(1.0) == -8


def _brute_block(x):
    """Definition by search: e is the integer with 2^(e+8) <= amax < 2^(e+9);
    each element is the E4M3 grid value (times 2^e) nearest to it, ties to the
    even mantissa, above the grid -> +-448 * 2^e."""
    amax = max(abs(v) for v in x)
    e = 0
    if amax > 0:
        e = -200
        while not (2.0 ** (e + 8) <= amax < 2.0 ** (e + 9)):
            e += 1
        e = max(-127, min(127, e))
    grid = [(O.e4m3_decode(np.uint8(c)).item(), c) for c in range(0x7F)]   # non-negative finite values
    out = []
    for v in x:
        a = abs(v) / 2.0 ** e
        if a >= 448.0:
            m = 448.0
        else:
            best = min(grid, key=lambda gc: (abs(gc[0] - a), gc[1] & 1))  # nearest, then even code
            m = best[0]
        out.append(math.copysign(m, v) * 2.0 ** e)
    return e, np.array(out)


def test_random_blocks_against_brute_force():
    rng = np.random.default_rng(11)
    for trial in range(300):
        scale = 2.0 ** rng.integers(-40, 40)
        x = rng.standard_normal(32) * scale
        if trial % 7 == 0:
            x[rng.integers(0, 32, 5)] = 0.0
        if trial % 11 == 0:                       # exact grid points and ties
            x = rng.integers(-448, 449, 32).astype(np.float64) * 2.0 ** -3
        e, want = _brute_block(x)
        codes, sc = O.mxfp8_quantize(x)
        assert int(sc[0]) - 127 == e
        got = O.mxfp8_dequantize(codes, sc)
        assert np.array_equal(np.abs(got), np.abs(want)), trial
        assert np.all((got == 0) | (np.sign(got) == np.sign(x)))


def test_error_bound_and_block_independence():
    rng = np.random.default_rng(12)
    x = rng.standard_normal((50, 128)) * 2.0 ** rng.integers(-20, 20, (50, 1))
    codes, sc = O.mxfp8_quantize(x)
    assert sc.shape == (50, 4)
    rec = O.mxfp8_dequantize(codes, sc)
    s = np.repeat(O.e8m0_decode(sc), 32, axis=1)
    sat = np.abs(x) / s > 448.0
    bound = np.maximum(np.abs(x) * 2.0 ** -4, s * 2.0 ** -10)     # half a 3-bit step, or half the subnormal step
    assert np.all(np.abs(rec - x)[~sat] <= bound[~sat])
    assert np.all(np.abs(rec[sat]) == 448.0 * s[sat])
    # one block's values do not move another block's codes
    y = x.copy()
    y[:, 32:64] *= 1000.0
    c2, s2 = O.mxfp8_quantize(y)
    keep = np.r_[0:32, 64:128]
    assert np.array_equal(c2[:, keep], codes[:, keep]) and np.array_equal(s2[:, [0, 2, 3]], sc[:, [0, 2, 3]])


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_hand_indexer_example_in_mxfp8_form():
    """The 4-token example, every vector padded with zeros to one block of 32:
    each q and k row is then an exact MXFP8 value, so the MXFP8 path must give
    the hand-expanded scores exactly."""
    ps, pt = HAND["page_size"], np.array(HAND["page_table"], np.int32)
    seqs = O.Seqs(ctx_len=np.array([4]), q_seq_start=np.array([0, 4]), page_table=pt, page_size=ps)
    q = np.zeros((4, 2, 32))
    q[:, :, :2] = HAND["qI"]
    k_log = np.zeros((4, 32))
    k_log[:, :2] = HAND["kI_logical"]
    codes_log, sc_log = O.mxfp8_quantize(k_log)
    assert np.array_equal(O.mxfp8_dequantize(codes_log, sc_log), k_log)
    codes = np.zeros((4, 32), np.uint8)
    sc = np.zeros((4, 1), np.uint8)
    for s in range(4):
        r = pt[0, s // ps] * ps + s % ps
        codes[r], sc[r] = codes_log[s], sc_log[s]
    got = O.index_scores(seqs, _bf16_bits(q), np.array(HAND["w"]), codes, sc)
    for t, row in enumerate(HAND["scores"]):
        assert np.array_equal(got[t], np.array(row, np.float64)), (t, got[t], row)


def test_mx_scores_equal_bf16_scores_on_the_dequantized_values():
    """Composition: the MXFP8 indexer is the bf16 formula applied to the
    exactly dequantized query and key rows (E4M3 values times powers of two are
    bf16 values, so the bf16 path sees the same numbers)."""
    rng = np.random.default_rng(13)
    ps, B, H, d = 4, 2, 3, 64
    ctx = np.array([9, 6])
    pages = (ctx + ps - 1) // ps
    pt = np.full((B, pages.max()), -1, np.int32)
    perm = rng.permutation(pages.sum())
    pt[0, : pages[0]] = perm[: pages[0]]
    pt[1, : pages[1]] = perm[pages[0]:]
    seqs = O.Seqs(ctx_len=ctx, q_seq_start=np.array([0, 9, 15]), page_table=pt, page_size=ps)
    R = pages.sum() * ps
    qf = rng.standard_normal((15, H, d)) * 2.0 ** rng.integers(-6, 6, (15, H, 1))
    qbits = _bf16_bits(qf)
    kc, ks = O.mxfp8_quantize(rng.standard_normal((R, d)) * 3.0)
    w = rng.standard_normal((15, H)) / 8
    got = O.index_scores(seqs, qbits, w, kc, ks)
    q_deq = O.mxfp8_dequantize(*O.mxfp8_quantize(O.bf16_to_f64(qbits)))
    k_deq = O.mxfp8_dequantize(kc, ks)
    assert np.array_equal(O.bf16_to_f64(_bf16_bits(q_deq)), q_deq)      # exact in bf16
    want = O.index_scores(seqs, _bf16_bits(q_deq), w, _bf16_bits(k_deq))
    for a, b in zip(got, want):
        assert np.array_equal(a, b)
    # and the query's group scales matter: scaling one block of a query row by
    # 2^10 moves that row's scores unless its dot products are all negative
    q2 = qf.copy()
    q2[0, 0, :32] *= 2.0 ** 10
    got2 = O.index_scores(seqs, _bf16_bits(q2), w, kc, ks, tokens=[0])
    assert not np.array_equal(got2[0], got[0])
