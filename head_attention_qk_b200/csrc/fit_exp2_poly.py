"""Fit the polynomial used by the kernels' software exp2.

The kernels compute 2^x for part of the softmax elements on the FMA pipe
instead of the MUFU unit, by Cody-Waite range reduction (the method of W. J.
Cody and W. Waite, "Software Manual for the Elementary Functions", 1980):
    j = floor(x),  f = x - j in [0, 1),  2^x = 2^j * p(f),
with 2^j applied by adding j to the exponent field of p(f).

p is the degree-n polynomial minimising the maximum relative error
|p(f) - 2^f| / 2^f over [0, 1], found here as a linear program over a dense
grid (scipy.optimize.linprog), and the coefficients are printed as C constants.

Usage: python fit_exp2_poly.py [degree ...]
"""
import sys

import numpy as np
from scipy.optimize import linprog


def fit(deg: int, n: int = 4001):
    f = np.linspace(0.0, 1.0, n)
    y = np.exp2(f)
    V = np.vander(f, deg + 1, increasing=True) / y[:, None]    # p(f)/2^f, linear in the coefficients
    # variables: c_0..c_deg, t ; minimise t subject to |V c - 1| <= t
    A = np.vstack([np.hstack([V, -np.ones((n, 1))]), np.hstack([-V, -np.ones((n, 1))])])
    b = np.concatenate([np.ones(n), -np.ones(n)])
    cost = np.zeros(deg + 2)
    cost[-1] = 1.0
    res = linprog(cost, A_ub=A, b_ub=b, bounds=[(None, None)] * (deg + 2), method="highs")
    if not res.success:
        raise RuntimeError(res.message)
    c = res.x[:-1]
    # error of the fp32-rounded coefficients on a finer grid
    cf = c.astype(np.float32).astype(np.float64)
    g = np.linspace(0.0, 1.0, 200001)
    err = np.max(np.abs(np.polyval(cf[::-1], g) / np.exp2(g) - 1.0))
    return cf, err


def main(argv):
    degs = [int(a) for a in argv] or [3, 4]
    for d in degs:
        c, err = fit(d)
        print("// degree %d, max relative error %.3e" % (d, err))
        print("constexpr float kExp2PolyDeg%d[%d] = {%s};" % (d, d + 1, ", ".join("%.9ef" % x for x in c)))


if __name__ == "__main__":
    main(sys.argv[1:])
