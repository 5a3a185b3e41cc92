"""Pins of the oracle's Top-K against a brute-force rank count (position s is
chosen iff fewer than K positions beat it, where s' beats s when its score is
larger, or equal with s' < s), exhaustively on tiny tie-heavy inputs."""
import itertools

import numpy as np

from oracle import dsa_oracle as O


def _rank_count(scores, K):
    n = len(scores)
    chosen = []
    for s in range(n):
        beat = 0
        for s2 in range(n):
            if scores[s2] > scores[s] or (scores[s2] == scores[s] and s2 < s):
                beat += 1
        if beat < K:
            chosen.append(s)
    return chosen + [-1] * (K - len(chosen))


def test_exhaustive_tiny_tie_heavy():
    # every score vector over a 3-value alphabet up to length 7, every K
    alphabet = [-1.0, 0.0, 2.5]
    for n in range(1, 8):
        for vals in itertools.product(alphabet, repeat=n):
            for K in range(1, n + 2):
                assert O.topk_select(np.array(vals), K).tolist() == _rank_count(list(vals), K)


def test_random_small_rows_all_K():
    rng = np.random.default_rng(5)
    for _ in range(300):
        n = int(rng.integers(1, 13))
        kind = rng.integers(0, 3)
        if kind == 0:
            v = rng.standard_normal(n).astype(np.float32).astype(np.float64)
        elif kind == 1:
            v = rng.integers(-2, 3, n).astype(np.float64)
        else:
            v = rng.choice([-0.0, 0.0, 1.0, -1.0], n)
        for K in range(1, 14):
            assert O.topk_select(v, K).tolist() == _rank_count(list(v), K)


def test_signed_zero_is_one_value():
    v = np.array([-0.0, 0.0, -0.0, 0.0])
    assert O.topk_select(v, 2).tolist() == [0, 1]
    v = np.array([0.0, -0.0, -1.0, -0.0])
    assert O.topk_select(v, 3).tolist() == [0, 1, 3]


def test_distinct_values_match_library_sort():
    rng = np.random.default_rng(6)
    for n, K in [(5000, 2048), (300, 256), (2048, 2048), (2049, 2048)]:
        v = rng.permutation(n).astype(np.float64) * 0.37 - 11.0
        ref = np.sort(np.argsort(-v, kind="stable")[:K])
        got = O.topk_select(v, K)
        assert np.array_equal(got[: min(K, n)], ref)


def test_nan_rejected():
    try:
        O.topk_select(np.array([1.0, np.nan]), 1)
    except ValueError:
        return
    raise AssertionError("NaN accepted")
