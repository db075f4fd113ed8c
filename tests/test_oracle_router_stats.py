"""Pins of the oracle's router statistics ("MoE (Mixture-of-Experts) 算法介绍",
第三部分: router z-loss on the L2 norm of the logits, gate entropy).

Closed forms: equal logits give the entropy ln n; two experts with logits
a, b give the binary entropy of sigmoid(a - b); the z-loss of d = 1 rows is
the sum of squared weights times x^2.  scipy's entropy of numpy's softmax is
an independent library check on random rows, and the forward pass reports
their means over tokens in losses[8], losses[9]."""
import math

import numpy as np
import pytest
from scipy.special import softmax
from scipy.stats import entropy

from oracle import oracle as O


def _stats(x, Wg, bg=None):
    T, d = x.shape
    n = Wg.shape[1]
    cfg = dict(T=T, d=d, n=n, k=1, f=8, noise=0)
    return O.router_stats(cfg, dict(x=x.astype(np.float32), Wg=Wg.astype(np.float32),
                                    bg=None if bg is None else bg.astype(np.float32)))


def test_equal_logits_give_log_n():
    for n in (1, 2, 7, 256):
        z, h = _stats(np.ones((3, 1)), np.full((1, n), 0.5))
        assert h == pytest.approx(3 * math.log(n), abs=1e-12)
        assert z == pytest.approx(3 * n * 0.25, abs=1e-12)


def test_two_experts_binary_entropy():
    a, b = 1.25, -0.5
    p = 1.0 / (1.0 + math.exp(-(a - b)))
    want = -(p * math.log(p) + (1 - p) * math.log(1 - p))
    z, h = _stats(np.array([[1.0]]), np.array([[a, b]]))
    assert h == pytest.approx(want, abs=1e-12)
    assert z == pytest.approx(a * a + b * b, abs=1e-12)


def test_bias_enters_the_logits():
    # x = 0: the logits are the bias alone
    z, h = _stats(np.zeros((2, 3)), np.ones((3, 2)), bg=np.array([3.0, -4.0]))
    assert z == pytest.approx(2 * 25.0, abs=1e-12)


def test_random_rows_against_scipy():
    rng = np.random.default_rng(5)
    x = rng.normal(0, 1, (40, 12)).astype(np.float32)
    Wg = rng.normal(0, 0.7, (12, 9)).astype(np.float32)
    z, h = _stats(x, Wg)
    c = x.astype(np.float64) @ Wg.astype(np.float64)
    assert h == pytest.approx(sum(entropy(softmax(r)) for r in c), rel=1e-12)
    assert z == pytest.approx(float((c * c).sum()), rel=1e-12)


def test_forward_reports_means_only_when_asked():
    rng = np.random.default_rng(1)
    T, d, n, f = 10, 8, 4, 8
    inp = dict(x=rng.normal(0, 1, (T, d)).astype(np.float32),
               Wg=rng.normal(0, 1, (d, n)).astype(np.float32),
               Wn=rng.normal(0, 1, (d, n)).astype(np.float32),
               W1=rng.normal(0, 0.3, (n, f, d)).astype(np.float32),
               W2=rng.normal(0, 0.3, (n, d, f)).astype(np.float32))
    cfg = dict(T=T, d=d, n=n, k=2, f=f)
    assert np.all(O.forward(cfg, inp)["losses"][8:] == 0.0)
    z, h = O.router_stats(cfg, inp)
    out = O.forward(dict(cfg, router_stats=1), inp)
    assert out["losses"][8] == pytest.approx(z / T, rel=1e-15)
    assert out["losses"][9] == pytest.approx(h / T, rel=1e-15)
