"""dsa_topk against the oracle on identical fp32 scores: bit-exact index arrays."""
import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O

pytestmark = pytest.mark.gpu


def _run(lib, scores_np, row_len_np, K):
    scores = torch.from_numpy(scores_np).cuda()
    row_len = torch.from_numpy(row_len_np.astype(np.int32)).cuda()
    idx = lib.dsa_topk(scores, row_len, K).cpu().numpy()
    for t in range(scores_np.shape[0]):
        ref = O.topk_select(scores_np[t, : row_len_np[t]], K)
        assert np.array_equal(idx[t], ref), (t, int(row_len_np[t]), K,
                                              np.nonzero(idx[t] != ref)[0][:8])


def test_random_rows_all_lengths(lib):
    rng = np.random.default_rng(0)
    T, ld = 24, 5004
    s = rng.standard_normal((T, ld)).astype(np.float32)
    lens = rng.integers(1, ld + 1, T)
    lens[:4] = [1, 255, 256, 257]
    for K in (1, 7, 256, 2048):
        _run(lib, s, lens, K)


def test_ties_and_signed_zero(lib):
    rng = np.random.default_rng(1)
    T, ld = 16, 3000
    s = rng.integers(-2, 3, (T, ld)).astype(np.float32)
    s[s == 0] = np.where(rng.random(np.count_nonzero(s == 0)) < 0.5, -0.0, 0.0).astype(np.float32)
    s[3] = 1.5                                    # one value everywhere
    s[4] = -0.0
    s[5, ::2] = 0.0
    s[5, 1::2] = -0.0
    lens = np.full(T, ld)
    lens[6] = 2047
    lens[7] = 2048
    lens[8] = 2049
    for K in (1, 100, 2048):
        _run(lib, s, lens, K)


def test_index_like_distributions(lib):
    rng = np.random.default_rng(2)
    # ReLU-sum-like rows: a spike of exact zeros, a positive tail, a few planted
    T, ld = 8, 131072
    s = np.maximum(rng.standard_normal((T, ld)), 0).astype(np.float32) * rng.random((T, ld)).astype(np.float32)
    s[:, rng.choice(ld, 64, replace=False)] += 50.0
    s[2] = np.abs(s[2])
    s[3, :100000] = 0.0
    _run(lib, s, np.full(T, ld), 2048)
    # causal prefill rows of a long sequence
    T, ld = 48, 32768
    s = (rng.standard_normal((T, ld)) * 3).astype(np.float32)
    lens = np.sort(rng.integers(1, ld + 1, T))
    _run(lib, s, lens, 2048)


def test_denormals_and_extremes(lib):
    rng = np.random.default_rng(3)
    T, ld = 6, 4096
    s = (rng.standard_normal((T, ld)) * 1e-40).astype(np.float32)   # subnormals
    s[1] = rng.choice(np.array([np.float32(3.0e38), np.float32(-3.0e38), np.float32(1e-45)]), ld)
    s[2] = np.float32(np.inf)
    s[2, ::3] = -np.inf
    _run(lib, s, np.full(T, ld), 1000)


def _low_bits_row(rng, n, distinct):
    """Values that share their top 22 key bits and differ in the low 10 only."""
    return (np.float32(1.0) + rng.integers(0, distinct, n).astype(np.float32) * np.float32(2.0 ** -23)).astype(
        np.float32)


def test_degenerate_threshold_bins(lib):
    rng = np.random.default_rng(4)
    # few rows (several CTAs per row): rows whose kept pairs overflow shared memory
    T, ld = 8, 40000
    s = rng.standard_normal((T, ld)).astype(np.float32)
    s[0] = 2.0                                          # one value everywhere
    s[1] = rng.integers(0, 3, ld).astype(np.float32)    # three values, ties at the threshold
    s[2] = _low_bits_row(rng, ld, 1024)                 # digit 3 decides, with ties
    s[3] = _low_bits_row(rng, ld, 7)
    s[4, :] = 0.0
    s[4, rng.choice(ld, 5000, replace=False)] = 1.0     # threshold inside the exact ones
    s[5] = np.where(rng.random(ld) < 0.5, np.float32(1.0), np.float32(1.0 + 2.0 ** -22))
    lens = np.full(T, ld)
    lens[6] = 9000
    for K in (2048, 1000):
        _run(lib, s, lens, K)
    # many rows (one CTA per row): kept pairs beyond the one-CTA stage
    T, ld = 300, 16384
    s = rng.standard_normal((T, ld)).astype(np.float32)
    s[0] = 7.0
    s[1] = rng.integers(0, 2, ld).astype(np.float32)
    s[2] = _low_bits_row(rng, ld, 1024)
    s[3] = _low_bits_row(rng, ld, 3)
    s[4:8] = np.float32(1.0) + (rng.standard_normal((4, ld)) * 1e-3).astype(np.float32)
    _run(lib, s, np.full(T, ld), 2048)
