"""Constants written into the CUDA sources, checked on the CPU against the
mathematics they come from (their use is covered by the GPU parity tests;
these catch a mistyped digit before a GPU run)."""
import math
import os
import re

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "selective_state_space_50_b200", "csrc")


def _consts(path, names):
    src = open(os.path.join(CSRC, path)).read()
    out = {}
    for n in names:
        m = re.search(r"constexpr float " + n + r" = ([0-9.eE+-]+)f;", src)
        assert m, n
        out[n] = float(m.group(1))
    return out


def test_zoh_series_coefficients_in_arg_units():
    """φ(x) = Σ x^k/(k+1)!, evaluated in arg = x log2(e): the coefficient of
    arg^k is ln(2)^k/(k+1)!; the switch |x| < 0.1 is |arg| < 0.1 log2(e)."""
    c = _consts("ssm_common.cuh", ["L1", "L2", "L3", "L4", "L5", "kSmall"])
    for k in range(1, 6):
        want = math.log(2.0) ** k / math.factorial(k + 1)
        assert abs(c[f"L{k}"] - want) <= 2e-7 * want, (k, c[f"L{k}"], want)
    assert abs(c["kSmall"] - 0.1 / math.log(2.0)) <= 1e-7


def test_zoh_series_accuracy_over_its_range():
    """With those coefficients the degree-5 series in arg stays within its
    truncation error (x^6/7! < 3e-10 for |x| < 0.1) of φ over its range."""
    c = _consts("ssm_common.cuh", ["L1", "L2", "L3", "L4", "L5", "kSmall"])
    arg = np.linspace(-c["kSmall"], c["kSmall"], 2001)
    x = arg * math.log(2.0)
    exact = np.where(x == 0, 1.0, np.expm1(x) / np.where(x == 0, 1.0, x))
    ser = 1 + arg * (c["L1"] + arg * (c["L2"] + arg * (c["L3"] + arg * (c["L4"] + arg * c["L5"]))))
    assert np.max(np.abs(ser - exact) / exact) < 5e-9


def test_zoh_psi_series_coefficients_and_accuracy():
    """ψ(x) = (x e^x - (e^x - 1))/x² = Σ x^k (k+1)/(k+2)!, evaluated in
    arg = x log2(e): the coefficient of arg^k is ln(2)^k (k+1)/(k+2)!; the
    degree-4 series stays within its truncation error (below 2e-8) of ψ for
    |x| < 0.1."""
    c = _consts("ssm_common.cuh", ["M1", "M2", "M3", "M4", "kSmallPsi"])
    for k in range(1, 5):
        want = math.log(2.0) ** k * (k + 1) / math.factorial(k + 2)
        assert abs(c[f"M{k}"] - want) <= 2e-7 * want, (k, c[f"M{k}"], want)
    assert abs(c["kSmallPsi"] - 0.1 / math.log(2.0)) <= 1e-7
    arg = np.linspace(-c["kSmallPsi"], c["kSmallPsi"], 2001)
    x = arg * math.log(2.0)
    xs = np.where(x == 0, 1.0, x)
    exact = np.where(x == 0, 0.5, (x * np.exp(x) - np.expm1(x)) / (xs * xs))
    ser = 0.5 + arg * (c["M1"] + arg * (c["M2"] + arg * (c["M3"] + arg * c["M4"])))
    assert np.max(np.abs(ser - exact) / exact) < 5e-8


def test_log1p_polynomial_of_the_one_sfu_softplus():
    """log1p_poly2: x q(x) with q fitted to log1p(x)/x on [0, 1]; evaluated in
    fp32 Horner form it stays within 3e-7 relative of log1p over [0, 1], and
    the softplus built on it, max(r, 0) + log1p(e^-|r|), within 4e-7 relative
    of the exact softplus over r in [-30, 30] (e^-|r| taken exactly here)."""
    src = open(os.path.join(CSRC, "ssm_common.cuh")).read()
    q = []
    for k in range(9):
        m = re.search(r"Q%d = ([0-9.eE+-]+)f" % k, src)
        assert m, k
        q.append(np.float32(float(m.group(1))))

    def poly(x32):
        acc = np.full_like(x32, q[8])
        for k in range(7, -1, -1):
            acc = (acc * x32 + q[k]).astype(np.float32)
        return (x32 * acc).astype(np.float32)

    x = np.linspace(0.0, 1.0, 100001).astype(np.float32)
    ref = np.log1p(x.astype(np.float64))
    got = poly(x).astype(np.float64)
    rel = np.abs(got - ref) / np.where(ref == 0, 1.0, ref)
    assert rel.max() < 3e-7, rel.max()
    r = np.linspace(-30.0, 30.0, 200001)
    e = np.exp(-np.abs(r)).astype(np.float32)
    sp = (np.maximum(r, 0.0).astype(np.float32) + poly(e)).astype(np.float64)
    exact = np.logaddexp(0.0, r)
    assert (np.abs(sp - exact) / exact).max() < 4e-7
