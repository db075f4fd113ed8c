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
    # u1 = 1 (top 24 bits of w0 all ones) -> sqrt(-2 ln 1) = 0
    assert orc.box_muller(0xFFFFFFFF, 0x12345678) == 0.0
    # u2 = 0 -> cos 0 = 1: eps = sqrt(-2 ln u1); w0 = 0 -> u1 = 2^-24
    assert orc.box_muller(0, 0) == pytest.approx(math.sqrt(48 * math.log(2)), rel=1e-15)
    # u2 = 1/2 -> cos(pi) = -1
    assert orc.box_muller(0, 0x80000000) == pytest.approx(-math.sqrt(48 * math.log(2)), rel=1e-15)
    # u2 = 1/4 -> cos(pi/2) = 0
    assert abs(orc.box_muller(0, 0x40000000)) < 1e-15
    # u1 = 1/2 exactly: w0 >> 8 = 2^23 - 1
    assert orc.box_muller((2**23 - 1) << 8, 0) == pytest.approx(math.sqrt(2 * math.log(2)), rel=1e-15)


def test_noise_stream_convention(orc):
    """The even expert of a pair takes Philox words (0,1), the odd one (2,3),
    with counter (token, expert/2, gate, 0) and key (seed lo, seed hi)."""
    seed = 0x0123456789ABCDEF
    for t, e, g in [(0, 0, 0), (5, 7, 0), (123, 4094, 3), (65535, 4095, 64)]:
        w = orc.philox4x32_10([t, e >> 1, g, 0], [seed & 0xFFFFFFFF, seed >> 32])
        want = orc.box_muller(int(w[0]), int(w[1])) if e % 2 == 0 else orc.box_muller(int(w[2]), int(w[3]))
        assert orc.noise(seed, t, e, g) == want


def test_noise_is_standard_normal(orc):
    vals = np.array([orc.noise(0, t, e, 0) for t in range(500) for e in range(200)])
    N = vals.size
    assert abs(vals.mean()) < 5 / math.sqrt(N)
    assert abs(vals.var() - 1.0) < 5 * math.sqrt(2.0 / N)
    assert scipy.stats.kstest(vals, "norm").pvalue > 1e-4
    # even/odd partners come from disjoint words: no correlation
    ev = vals.reshape(500, 100, 2)
    r = np.corrcoef(ev[..., 0].ravel(), ev[..., 1].ravel())[0, 1]
    assert abs(r) < 5 / math.sqrt(ev[..., 0].size)
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
