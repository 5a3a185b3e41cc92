"""Pins of the oracle's number formats against torch's own float8_e4m3fn and
bfloat16 conversions (library routines), plus the saturation rule."""
import numpy as np
import torch

from oracle import dsa_oracle as O


def test_e4m3_decode_all_codes_match_torch():
    codes = np.arange(256, dtype=np.uint8)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.e4m3_decode(codes)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
    # sign of zero is kept
    assert np.signbit(got[0x80]) and not np.signbit(got[0x00])
    assert O.e4m3_decode(np.array([0x7E]))[0] == 448.0
    assert O.e4m3_decode(np.array([0x01]))[0] == 2.0 ** -9


def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_encode_matches_torch_below_saturation():
    vals = O.e4m3_decode(np.arange(0x7F, dtype=np.uint8))          # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2                               # exact ties
    f32 = mids.astype(np.float32)
    assert np.array_equal(f32.astype(np.float64), mids)            # ties are fp32-exact
    up = np.nextafter(f32, np.float32(np.inf))
    dn = np.nextafter(f32, np.float32(-np.inf))
    rng = np.random.default_rng(0)
    rnd = rng.uniform(-463.9, 463.9, 200_000).astype(np.float32)
    small = (rng.standard_normal(50_000) * 2.0 ** rng.integers(-20, 0, 50_000)).astype(np.float32)
    x = np.concatenate([vals, -vals, mids, -mids, up, dn, -up, -dn, rnd, small,
                        np.array([0.0, -0.0, 448.0, 463.9, -463.9], np.float32)]).astype(np.float32)
    x = x[np.abs(x) < 464.0]
    got = O.e4m3_encode(x.astype(np.float64))
    ref = _torch_e4m3(x)
    bad = np.nonzero(got != ref)[0]
    assert bad.size == 0, (x[bad[:5]], got[bad[:5]], ref[bad[:5]])


def test_e4m3_encode_saturates():
    x = np.array([448.0, 464.0, 500.0, 1e6, 3e38, -464.0, -1e30])
    got = O.e4m3_encode(x)
    assert list(got) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert O.e4m3_encode(np.array([np.nan]))[0] == 0x7F


def test_bf16_decode_all_patterns_match_torch():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ref = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()
    got = O.bf16_to_f64(bits)
    assert np.array_equal(np.isnan(ref), np.isnan(got))
    ok = ~np.isnan(ref)
    assert np.array_equal(ref[ok], got[ok])
