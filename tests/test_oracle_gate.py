"""Pins of the oracle's gate and smoothed-load estimator (CPU only).

Hand-computed cases, equivalences the pages state, library routines (numpy
sort, scipy softmax / Normal CDF) and a Monte-Carlo check of P(x,i).
"""
import math

import numpy as np
import pytest
import scipy.special
import scipy.stats


def sigmoid(z):
    return 1.0 / (1.0 + math.exp(-z))


def test_hand_k2_noise_off(orc):
    """n=4, d=2, integer W_g, no noise, k=2.
    x = (1, 2); columns of W_g: (1,0), (0,1), (2,1), (-1,3)
    -> logits (1, 2, 4, 5); kept = {3, 2}; g = (sigma(1), 1 - sigma(1))."""
    x = np.array([1.0, 2.0])
    Wg = np.array([[1.0, 0.0, 2.0, -1.0], [0.0, 1.0, 1.0, 3.0]])
    r = orc.gate_row(x, Wg, 2, noise=False)
    assert list(r["H"]) == [1.0, 2.0, 4.0, 5.0]
    assert list(r["idx"]) == [3, 2]
    assert r["gates"][0] == pytest.approx(sigmoid(1.0), rel=1e-15)
    assert r["gates"][1] == pytest.approx(1.0 - sigmoid(1.0), rel=1e-14)


def test_hand_bias_is_part_of_clean_logit(orc):
    x = np.array([1.0, 2.0])
    Wg = np.array([[1.0, 0.0, 2.0, -1.0], [0.0, 1.0, 1.0, 3.0]])
    r = orc.gate_row(x, Wg, 2, bg=np.array([10.0, 0.0, 0.0, 0.0]), noise=False)
    assert list(r["c"]) == [11.0, 2.0, 4.0, 5.0]
    assert list(r["idx"]) == [0, 3]
    assert r["gates"][0] == pytest.approx(sigmoid(6.0), rel=1e-14)


def test_hand_exact_tie_lower_index_wins(orc):
    """logits (3, 3, 1, 3), k=2 -> experts 0 and 1, gates 1/2 each."""
    x = np.array([1.0])
    Wg = np.array([[3.0, 3.0, 1.0, 3.0]])
    r = orc.gate_row(x, Wg, 2, noise=False)
    assert list(r["idx"]) == [0, 1]
    assert list(r["order"]) == [0, 1, 3, 2]
    assert list(r["gates"]) == [0.5, 0.5]


def test_hand_switch_router(orc):
    """Switch router, n=3: logits (0, ln 2, ln 3) -> p = (1/6, 2/6, 3/6);
    the token goes to expert 2 with gate p_2 = 1/2 (no renormalisation)."""
    x = np.array([1.0])
    Wg = np.array([[0.0, math.log(2.0), math.log(3.0)]], np.float32)
    r = orc.gate_row(x, Wg, 1, router=1, noise=False)
    assert list(r["idx"]) == [2]
    assert r["gates"][0] == pytest.approx(0.5, rel=1e-7)
    assert r["p"] == pytest.approx([1 / 6, 2 / 6, 3 / 6], rel=1e-7)


def test_topk_order_matches_numpy_lexsort(orc):
    rng = np.random.default_rng(3)
    for trial in range(30):
        d, n = 16, int(rng.integers(2, 70))
        k = int(rng.integers(1, min(n, 8) + 1))
        x = rng.standard_normal(d)
        Wg = rng.standard_normal((d, n)) / 4
        if trial % 3 == 0:  # force exact ties
            Wg[:, 1::3] = Wg[:, 0:1]
        Wn = rng.standard_normal((d, n)) / 4
        r = orc.gate_row(x, Wg, k, Wn=Wn, seed=trial, token=trial * 7)
        H = r["H"]
        want = np.lexsort((np.arange(n), -H.astype(np.float64)))
        assert np.array_equal(r["order"], want)
        # softmax over the kept k == softmax over all then renormalised over
        # the kept (the two forms the pages give for the same gate)
        full = scipy.special.softmax(H.astype(np.float64))
        ren = full[want[:k]] / full[want[:k]].sum()
        assert r["gates"] == pytest.approx(ren, rel=1e-12)
        # KeepTopK then softmax: -inf entries get exactly 0
        kt = np.full(n, -np.inf)
        kt[want[:k]] = H[want[:k]]
        dense = scipy.special.softmax(kt)
        assert dense[want[:k]] == pytest.approx(r["gates"], rel=1e-12)
        assert float(np.sum(r["gates"])) == pytest.approx(1.0, abs=1e-15 * k)


def test_clean_and_noise_logits_match_library_matmul(orc):
    rng = np.random.default_rng(4)
    d, n = 24, 40
    x = rng.standard_normal(d).astype(np.float32)
    Wg = rng.standard_normal((d, n)).astype(np.float32)
    Wn = rng.standard_normal((d, n)).astype(np.float32)
    bg = rng.standard_normal(n).astype(np.float32)
    r = orc.gate_row(x, Wg, 3, bg=bg, Wn=Wn, seed=11, token=9)
    c = x.astype(np.float64) @ Wg.astype(np.float64) + bg
    s = np.logaddexp(0.0, x.astype(np.float64) @ Wn.astype(np.float64))
    assert r["c"] == pytest.approx(c, rel=1e-12, abs=1e-12)
    assert r["s"] == pytest.approx(s, rel=1e-12, abs=1e-300)
    eps = np.array([orc.noise(11, 9, i, 0) for i in range(n)])
    # H is the fp64 value rounded once to fp32 (summation order may move the
    # fp64 value by an ulp of fp64, hence one fp32 ulp of slack)
    np.testing.assert_allclose(r["H"], (c + eps * s).astype(np.float32), rtol=1.2e-7, atol=1e-30)


def _kth_excluding_bruteforce(H, k, i):
    rest = np.sort(np.delete(H.astype(np.float64), i))[::-1]
    return rest[k - 1] if k - 1 < rest.size else -np.inf


def test_load_row_matches_bruteforce_kth_excluding(orc):
    rng = np.random.default_rng(5)
    for trial in range(20):
        n = int(rng.integers(2, 40))
        k = int(rng.integers(1, min(n, 6) + 1))
        c = rng.standard_normal(n)
        s = np.abs(rng.standard_normal(n)) + 0.1
        H = (c + rng.standard_normal(n) * s).astype(np.float32)
        P = orc.load_row(c, s, H, k)
        want = [scipy.stats.norm.cdf((c[i] - _kth_excluding_bruteforce(H, k, i)) / s[i]) for i in range(n)]
        assert P == pytest.approx(want, rel=1e-12, abs=1e-300)


def test_load_row_special_values(orc):
    # k = n: nothing left to compete with -> P = 1 for every expert
    c = np.array([0.3, -1.0, 2.0]); s = np.ones(3); H = np.array([1.0, 0.0, 2.0], np.float32)
    assert list(orc.load_row(c, s, H, 3)) == [1.0, 1.0, 1.0]
    # clean logit exactly at the threshold -> Phi(0) = 1/2
    H = np.array([5.0, 3.0, 1.0], np.float32)   # k = 1: experts 1, 2 compare against 5
    c = np.array([0.0, 5.0, 5.0]); s = np.array([1.0, 2.0, 3.0])
    P = orc.load_row(c, s, H, 1)
    assert P[1] == 0.5 and P[2] == 0.5
    # expert 0 compares against the 2nd largest (3): Phi((0-3)/1)
    assert P[0] == pytest.approx(scipy.stats.norm.cdf(-3.0), rel=1e-12)
    # no noise: the indicator of being kept
    assert list(orc.load_row(c, s, H, 1, noise=False)) == [1.0, 0.0, 0.0]


def test_load_monte_carlo(orc):
    """P(x,i) is the probability that expert i is kept when only its own
    noise is redrawn, the other experts' noisy logits held fixed."""
    rng = np.random.default_rng(6)
    n, k = 12, 3
    c = rng.standard_normal(n)
    s = np.abs(rng.standard_normal(n)) + 0.2
    H = (c + rng.standard_normal(n) * s).astype(np.float32)
    P = orc.load_row(c, s, H, k)
    M = 400_000
    for i in (0, 5, 11):
        others = np.delete(H.astype(np.float64), i)
        kth = np.sort(others)[::-1][k - 1]
        draws = c[i] + rng.standard_normal(M) * s[i]
        # kept iff it beats the k-th largest of the others
        freq = np.mean(draws > kth)
        sigma = math.sqrt(max(P[i] * (1 - P[i]), 1e-12) / M)
        assert abs(freq - P[i]) < 5 * sigma + 1e-9, (i, freq, P[i])
