"""The routing kernels' Phi (csrc/phi.cuh), checked on the host.

The header's coefficients must be the ones csrc/phi_coef.py fits, and the
kernels' fp32 evaluation order applied to them must stay within 1e-6
relative of the standard normal CDF (scipy.special.ndtr, fp64) over the range
that reaches the smoothed load; the GPU parity tests then compare the load
itself with the oracle."""
import importlib.util
import os
import re

import numpy as np
from scipy.special import ndtr

CSRC = os.path.join(os.path.dirname(__file__), "..", "sparsely_gated_mixture_gate_b200", "csrc")


def _fit_module():
    spec = importlib.util.spec_from_file_location("phi_coef", os.path.join(CSRC, "phi_coef.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


def _header_coefficients():
    src = open(os.path.join(CSRC, "phi.cuh")).read()
    body = src[src.index("phi_cdf(float z)"):]
    first = float(re.search(r"float q = ([-0-9.e+]+)f;", body).group(1))
    rest = [float(v) for v in re.findall(r"q = fmaf\(q, t, ([-0-9.e+]+)f\);", body)]
    # Horner from the highest power down: reverse to t^0 first
    return np.array(([first] + rest)[::-1], dtype=np.float32)


def test_header_holds_the_fitted_coefficients():
    mod = _fit_module()
    fitted = mod.fit()
    header = _header_coefficients()
    assert header.shape == (mod.DEG + 1,)
    np.testing.assert_allclose(header, fitted, rtol=1e-6, atol=1e-9)
    assert "0.4f, x, 1.0f" in open(os.path.join(CSRC, "phi.cuh")).read() and mod.P == 0.4


def test_fp32_evaluation_tracks_the_normal_cdf():
    mod = _fit_module()
    c = _header_coefficients()
    z = np.linspace(-12.5, 8.0, 400001).astype(np.float32)
    ref = ndtr(z.astype(np.float64))
    got = mod.phi_fp32(z, c).astype(np.float64)
    assert np.max(np.abs(got - ref) / ref) < 1e-6
    # special values: symmetry point, the far tails, and the cut below -13.5
    assert abs(mod.phi_fp32(np.float32(0.0), c) - 0.5) < 1e-7
    assert mod.phi_fp32(np.float32(-14.0), c) == 0.0
    assert mod.phi_fp32(np.float32(30.0), c) == 1.0
    # monotone on a fine grid (a sign slip in a coefficient breaks this first)
    g = mod.phi_fp32(np.linspace(-9, 6, 20001).astype(np.float32), c)
    assert np.all(np.diff(g.astype(np.float64)) >= -1e-7 * g[1:])
