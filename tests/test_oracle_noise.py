"""Pins of the oracle's noise source and closed-form helpers (CPU only).

Every check compares the oracle with something other than itself: Triton's
own Philox (a library routine, run on the CPU interpreter), closed forms of
Box-Muller, scipy / numpy / torch routines, and distribution tests.
"""
import json
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import scipy.stats
import torch

HERE = os.path.dirname(os.path.abspath(__file__))


def _triton_philox(cases):
    env = dict(os.environ, TRITON_INTERPRET="1")
    out = subprocess.run([sys.executable, os.path.join(HERE, "philox_triton_ref.py"), json.dumps(cases)],
                         check=True, capture_output=True, text=True, env=env, timeout=600)
    return json.loads(out.stdout.strip().splitlines()[-1])


def test_philox_matches_triton_library(orc):
    rng = np.random.default_rng(7)
    cases = [[0, 0, 0, 0, 0], [2**64 - 1, 2**32 - 1, 2**32 - 1, 2**32 - 1, 2**32 - 1]]
    for _ in range(14):
        seed = int(rng.integers(0, 2**63))
        cases.append([seed] + [int(v) for v in rng.integers(0, 2**32, size=4)])
    ref = _triton_philox(cases)
    for (seed, c0, c1, c2, c3), want in zip(cases, ref):
        got = orc.philox4x32_10([c0, c1, c2, c3], [seed & 0xFFFFFFFF, seed >> 32])
        assert [int(v) for v in got] == want, (seed, c0, c1, c2, c3)


def test_box_muller_closed_forms(orc):
    r24 = math.sqrt(48 * math.log(2))  # w0 = 0 -> u1 = 2^-24 -> r = sqrt(-2 ln 2^-24)
    # u1 = 1 (top 24 bits of w0 all ones) -> r = 0 on both branches
    assert orc.box_muller(0xFFFFFFFF, 0x12345678, 0) == 0.0
    assert orc.box_muller(0xFFFFFFFF, 0x12345678, 1) == 0.0
    # u2 = 0: cos = 1, sin = 0
    assert orc.box_muller(0, 0, 0) == pytest.approx(r24, rel=1e-15)
    assert orc.box_muller(0, 0, 1) == 0.0
    # u2 = 1/2: cos = -1, sin = 0
    assert orc.box_muller(0, 0x80000000, 0) == pytest.approx(-r24, rel=1e-15)
    assert abs(orc.box_muller(0, 0x80000000, 1)) < 1e-14
    # u2 = 1/4: cos = 0, sin = 1
    assert abs(orc.box_muller(0, 0x40000000, 0)) < 1e-15
    assert orc.box_muller(0, 0x40000000, 1) == pytest.approx(r24, rel=1e-15)
    # u2 = 3/4: sin = -1
    assert orc.box_muller(0, 0xC0000000, 1) == pytest.approx(-r24, rel=1e-15)
    # u1 = 1/2 exactly: w0 >> 8 = 2^23 - 1
    assert orc.box_muller((2**23 - 1) << 8, 0, 0) == pytest.approx(math.sqrt(2 * math.log(2)), rel=1e-15)
    # the two branches lie on one circle of radius r
    for w0, w1 in [(123456789, 987654321), (2**31, 2**30 + 12345), (77, 2**32 - 1)]:
        c, s_ = orc.box_muller(w0, w1, 0), orc.box_muller(w0, w1, 1)
        r = math.sqrt(-2 * math.log(((w0 >> 8) + 1) / 2**24))
        assert c * c + s_ * s_ == pytest.approx(r * r, rel=1e-13)


def test_noise_stream_convention(orc):
    """Experts 4m..4m+3 share counter (token, m, gate, 0) under key (seed lo,
    seed hi): words (0,1) give the cosine / sine branches for 4m, 4m+1,
    words (2,3) those for 4m+2, 4m+3."""
    seed = 0x0123456789ABCDEF
    for t, e, g in [(0, 0, 0), (5, 7, 0), (123, 4094, 3), (65535, 4095, 64), (9, 1, 2), (9, 2, 2)]:
        w = orc.philox4x32_10([t, e >> 2, g, 0], [seed & 0xFFFFFFFF, seed >> 32])
        q = e % 4
        want = orc.box_muller(int(w[2 * (q // 2)]), int(w[2 * (q // 2) + 1]), q % 2)
        assert orc.noise(seed, t, e, g) == want


def test_noise_is_standard_normal(orc):
    vals = np.array([orc.noise(0, t, e, 0) for t in range(500) for e in range(200)])
    N = vals.size
    assert abs(vals.mean()) < 5 / math.sqrt(N)
    assert abs(vals.var() - 1.0) < 5 * math.sqrt(2.0 / N)
    assert scipy.stats.kstest(vals, "norm").pvalue > 1e-4
    # the cosine / sine partners and the two word pairs of one counter are
    # uncorrelated
    q = vals.reshape(500, 50, 4)
    for a, b in [(0, 1), (2, 3), (0, 2), (1, 3)]:
        r = np.corrcoef(q[..., a].ravel(), q[..., b].ravel())[0, 1]
        assert abs(r) < 5 / math.sqrt(q[..., 0].size)
    # cos^2 + sin^2 of one pair is a chi-square with 2 degrees of freedom
    r2 = (q[..., 0] ** 2 + q[..., 1] ** 2).ravel()
    assert scipy.stats.kstest(r2, "chi2", args=(2,)).pvalue > 1e-4
    # different gates / seeds give different deviates
    assert orc.noise(0, 3, 4, 0) != orc.noise(0, 3, 4, 1)
    assert orc.noise(0, 3, 4, 0) != orc.noise(1, 3, 4, 0)


def test_softplus(orc):
    assert orc.softplus(0.0) == pytest.approx(math.log(2), rel=1e-15)
    for z in np.linspace(-50, 50, 201):
        assert orc.softplus(float(z)) == pytest.approx(float(np.logaddexp(0.0, z)), rel=1e-13, abs=1e-300)
    assert orc.softplus(-745.0) >= 0.0


def test_phi(orc):
    assert orc.phi(0.0) == 0.5
    assert orc.phi(1.959963984540054) == pytest.approx(0.975, rel=1e-12)
    for z in np.linspace(-8, 8, 161):
        assert orc.phi(float(z)) == pytest.approx(float(scipy.stats.norm.cdf(z)), rel=1e-12, abs=1e-300)


def test_cv2(orc):
    assert orc.cv2([3.0, 3.0, 3.0, 3.0]) == 0.0
    assert orc.cv2([0.0, 2.0]) == pytest.approx(1.0)
    assert orc.cv2([1.0, 3.0]) == pytest.approx(0.25)
    assert orc.cv2([0.0, 0.0]) == 0.0
    v = np.random.default_rng(0).gamma(2.0, size=1000)
    assert orc.cv2(v) == pytest.approx(np.var(v) / np.mean(v) ** 2, rel=1e-12)


def test_bf16_round_matches_torch(orc):
    rng = np.random.default_rng(1)
    vals = np.concatenate([
        rng.standard_normal(4000).astype(np.float32) * 10,
        # exact ties: low 16 bits = 0x8000, even and odd bf16 mantissas
        (np.arange(1000, dtype=np.uint32) * 0x10000 + 0x3F808000).view(np.float32),
        np.array([0.0, -0.0, 1e-40, -1e-40, 3.4e38, np.inf, -np.inf], np.float32),
    ])
    want = torch.from_numpy(vals).to(torch.bfloat16).float().numpy()
    got = np.array([orc.bf16_round(float(v)) for v in vals], np.float32)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert math.isnan(orc.bf16_round(float("nan")))


def test_capacity(orc):
    # Switch workload: 32768 tokens / 128 experts * 1.25 = 320
    assert orc.capacity(32768, 1, 128, 1.25) == 320
    assert orc.capacity(3, 1, 2, 0.5) == 1          # ceil(0.75)
    assert orc.capacity(10, 2, 4, 1.0) == 5         # exact
    assert orc.capacity(10, 2, 3, 1.0) == 7         # ceil(6.67)
    assert orc.capacity(10, 2, 3, 0.0) == 2**63 - 1  # no limit
