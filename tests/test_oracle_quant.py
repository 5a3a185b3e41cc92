"""Pins of the index-query quantization: properties fixed by the format (the
scale is a power of two, nothing saturates, the scale is the tightest such
power, the error is within half an E4M3 step) and exact special cases."""
import numpy as np
import torch

from oracle import dsa_oracle as O


def _bf16_bits(x):
    t = torch.as_tensor(np.asarray(x, np.float32)).to(torch.bfloat16)
    return t.view(torch.int16).numpy().view(np.uint16)


def test_scale_is_tight_power_of_two_and_never_saturates():
    rng = np.random.default_rng(1)
    rows = rng.standard_normal((400, 64, 128)) * np.exp2(rng.integers(-30, 30, (400, 64, 1)))
    bits = _bf16_bits(rows)
    q = O.bf16_to_f64(bits)
    codes, sq = O.quantize_index_query(bits)
    m, e = np.frexp(sq)
    assert np.all(m == 0.5)                                  # exact powers of two
    amax = np.abs(q).max(-1)
    assert np.all(amax / sq <= 448.0)                        # no saturation
    assert np.all(amax / sq > 224.0)                         # a smaller scale would saturate
    # reconstruction: within half a step of the 3-bit mantissa (relative 2^-4),
    # or half the subnormal step 2^-10 * sq near zero
    rec = O.e4m3_decode(codes) * sq[..., None]
    err = np.abs(rec - q)
    bound = np.maximum(np.abs(q) * 2.0 ** -4, sq[..., None] * 2.0 ** -10)
    assert np.all(err <= bound)


def test_zero_row_and_exact_rows():
    x = np.zeros((1, 2, 4))
    x[0, 1] = [448.0, 1.0, -2.0, 0.5]          # E4M3 values, amax exactly 448 -> scale 1
    codes, sq = O.quantize_index_query(_bf16_bits(x))
    assert sq[0, 0] == 1.0 and np.all(codes[0, 0] == 0)
    assert sq[0, 1] == 1.0
    assert np.array_equal(O.e4m3_decode(codes[0, 1]), x[0, 1])
    y = x * 2.0                                 # amax 896 -> scale 2, same codes
    codes2, sq2 = O.quantize_index_query(_bf16_bits(y))
    assert sq2[0, 1] == 2.0 and np.array_equal(codes2[0, 1], codes[0, 1])
    z = x * 2.0 ** -5                           # amax 14 -> scale 2^-5
    codes3, sq3 = O.quantize_index_query(_bf16_bits(z))
    assert sq3[0, 1] == 2.0 ** -5 and np.array_equal(codes3[0, 1], codes[0, 1])


def test_pow2_exponent_boundaries():
    for e in range(-40, 40):
        b = 448.0 * 2.0 ** e
        assert O.pow2_exponent(b) == e
        assert O.pow2_exponent(np.nextafter(b, np.inf)) == e + 1
        assert O.pow2_exponent(np.nextafter(b, 0.0)) == e
    assert O.pow2_exponent(0.0) == 0
