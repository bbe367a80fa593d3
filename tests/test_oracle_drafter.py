"""Pins for oracle.drafter_topk (per-row log-softmax + top-k), each against
something other than the oracle's own formula: closed forms, invariants of
log-softmax and a brute-force sort."""
import itertools
import math

import numpy as np
import pytest

import oracle


def test_uniform_row_closed_form():
    # every probability is 1 / V
    for V in (1, 2, 7, 1000):
        lp, tk, st = oracle.drafter_topk(np.full((1, V), 3.25), min(V, 5))
        assert st[0] == oracle.OK
        assert np.allclose(lp[0], -math.log(V), rtol=0, atol=1e-6)
        assert list(tk[0]) == list(range(min(V, 5)))  # equal values: lower index first


def test_two_point_closed_form():
    # p(a) = 1 / (1 + e^(b - a))
    for a, b in ((0.0, 0.0), (1.5, -2.0), (-3.0, 4.0), (10.0, 10.5)):
        lp, tk, _ = oracle.drafter_topk(np.array([[a, b]]), 2)
        hi, lo = (a, b) if a >= b else (b, a)
        assert abs(lp[0, 0] - (-math.log1p(math.exp(lo - hi)))) < 1e-6
        assert abs(lp[0, 1] - (lo - hi - math.log1p(math.exp(lo - hi)))) < 1e-6
        assert tk[0, 0] == (0 if a >= b else 1)


def test_full_k_is_a_distribution():
    rng = np.random.default_rng(3)
    z = rng.standard_normal((4, 300)) * 4
    lp, tk, _ = oracle.drafter_topk(z, 300)
    for r in range(4):
        assert abs(math.fsum(math.exp(v) for v in lp[r].astype(np.float64)) - 1.0) < 1e-5
        assert sorted(tk[r].tolist()) == list(range(300))
        assert np.all(np.diff(lp[r]) <= 0)


def test_shift_invariance():
    rng = np.random.default_rng(4)
    z = np.round(rng.standard_normal((3, 64)) * 8) / 8  # exact in binary, with ties
    a = oracle.drafter_topk(z, 10)
    b = oracle.drafter_topk(z + 100.0, 10)
    assert np.array_equal(a[1], b[1])
    assert np.allclose(a[0], b[0], atol=2e-5, rtol=0)


@pytest.mark.parametrize("V,K", [(1, 1), (4, 2), (6, 6), (9, 3)])
def test_brute_force_order(V, K):
    rng = np.random.default_rng(V * 10 + K)
    for _ in range(20):
        z = rng.integers(-2, 3, size=V).astype(np.float64)  # many ties
        lp, tk, _ = oracle.drafter_topk(z[None], K)
        want = sorted(range(V), key=lambda i: (-z[i], i))[:K]
        assert tk[0].tolist() == want
        # the selected set beats every other index
        rest = [i for i in range(V) if i not in want]
        for i, j in itertools.product(want, rest):
            assert z[i] > z[j] or (z[i] == z[j] and i < j)
        assert np.all(np.diff(lp[0]) <= 0)


def test_non_finite_row_is_flagged_and_skipped():
    z = np.zeros((3, 8))
    z[1, 3] = np.nan
    z[2, 0] = np.inf
    lp, tk, st = oracle.drafter_topk(z, 4)
    assert list(st) == [oracle.OK, oracle.ERR_INPUT, oracle.ERR_INPUT]
    assert np.all(tk[1:] == -1) and np.all(np.isneginf(lp[1:]))
    assert np.all(tk[0] == np.arange(4))
