"""The kernels' software exp2 (Cody-Waite reduction + fitted cubic), emulated
step by step in float32 on the CPU with the constants read from sm100.cuh,
against exp2 in float64; and the constants against the fitting script."""
import os
import re
import sys

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "head_attention_qk_b200", "csrc")


def header_coeffs(deg=3):
    txt = open(os.path.join(CSRC, "sm100.cuh")).read()
    pat = r"kExp2C(\d) = ([0-9.e+-]+)f" if deg == 3 else r"kExp2D2C(\d) = ([0-9.e+-]+)f"
    vals = {int(m.group(1)): float(m.group(2)) for m in re.finditer(pat, txt)}
    return np.array([vals[i] for i in range(deg + 1)], dtype=np.float32)


def exp2_poly_emulated(x, deg=3):
    c = header_coeffs(deg)
    x = np.maximum(x.astype(np.float32), np.float32(-120.0))
    t = (np.floor(x.astype(np.float64)) + 12582912.0).astype(np.float32)      # round-down add of 1.5*2^23
    jf = (t.astype(np.float64) - 12582912.0).astype(np.float32)
    f = (x.astype(np.float64) - jf.astype(np.float64)).astype(np.float32)     # fma(jf, -1, x)
    p = c[deg]
    for k in range(deg - 1, -1, -1):                                          # Horner with fused multiply-add
        p = (p.astype(np.float64) * f.astype(np.float64) + np.float64(c[k])).astype(np.float32)
    bits = (p.view(np.uint32).astype(np.uint64) + t.view(np.uint32).astype(np.uint64) * 8388608) & 0xFFFFFFFF
    return bits.astype(np.uint32).view(np.float32)


@pytest.mark.parametrize("deg,bound", [(3, 1.0e-4), (2, 2.0e-3)])
def test_relative_error_over_softmax_range(deg, bound):
    x = np.linspace(-100.0, 8.5, 2_000_001, dtype=np.float64).astype(np.float32)
    got = exp2_poly_emulated(x, deg).astype(np.float64)
    ref = np.exp2(x.astype(np.float64))
    rel = np.abs(got / ref - 1.0)
    assert rel.max() < bound, rel.max()


@pytest.mark.parametrize("deg", [2, 3])
def test_underflow_is_clamped_not_wrapped(deg):
    x = np.array([-np.inf, -1e30, -500.0, -130.0, -120.5, -119.9], dtype=np.float32)
    got = exp2_poly_emulated(x, deg)
    assert np.all(np.isfinite(got)) and np.all(got >= 0) and np.all(got < 2.0 ** -118)


def test_header_constants_are_the_fitted_ones():
    sys.path.insert(0, CSRC)
    try:
        import fit_exp2_poly
    finally:
        sys.path.pop(0)
    for deg, bound in ((3, 1e-4), (2, 2e-3)):
        c, err = fit_exp2_poly.fit(deg)
        np.testing.assert_allclose(header_coeffs(deg), c.astype(np.float32), rtol=1e-6)
        assert err < bound
