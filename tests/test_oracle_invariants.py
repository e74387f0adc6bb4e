"""More pins for the CPU fp64 oracle: properties the mathematics of attention
fixes, chosen so that a plausible slip (a wrong normaliser, a missing scale,
a sign error or a transposed operand in the backward) breaks one of them.

Forward: O is a convex combination of the visible V rows (inside their
per-column hull), max score <= LSE <= max score + ln(number of visible
keys), O is linear in V, and moving every key by one vector c moves each
row's scores by the same amount (P unchanged, LSE + scale * q.c).
Backward: the rows of dS sum to zero (sum_j P_ij (dP_ij - Delta_i) = 0), so
dK summed over keys vanishes; the rows of P sum to one, so dV summed over
keys equals dO summed over the rows that see them.
"""
import math

import numpy as np
import pytest

pytestmark = pytest.mark.filterwarnings("ignore")


def rnd(shape, seed, s=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * s


def visible(Sq, Sk, causal):
    """[Sq, Sk] mask of the keys each query sees (bottom-right causal)."""
    if not causal:
        return np.ones((Sq, Sk), dtype=bool)
    return np.arange(Sk)[None, :] <= np.arange(Sq)[:, None] + (Sk - Sq)


@pytest.mark.parametrize("causal", [False, True])
def test_output_in_value_hull_and_lse_bounds(oracle_mod, causal):
    B, Hq, Hkv, Sq, Sk, D = 2, 4, 2, 19, 33, 16
    q, k, v = rnd((B, Hq, Sq, D), 101, 2.0), rnd((B, Hkv, Sk, D), 102), rnd((B, Hkv, Sk, D), 103)
    scale = 0.3
    o, lse = oracle_mod.attn_fwd(q, k, v, scale, causal=causal)
    vis = visible(Sq, Sk, causal)
    G = Hq // Hkv
    for b in range(B):
        for h in range(Hq):
            kk, vv = k[b, h // G], v[b, h // G]
            s = scale * q[b, h] @ kk.T
            for i in range(Sq):
                cols = vis[i]
                lo, hi = vv[cols].min(axis=0), vv[cols].max(axis=0)
                assert np.all(o[b, h, i] >= lo - 1e-12) and np.all(o[b, h, i] <= hi + 1e-12)
                smax = s[i, cols].max()
                assert smax - 1e-12 <= lse[b, h, i] <= smax + math.log(cols.sum()) + 1e-12


def test_linear_in_v(oracle_mod):
    q, k = rnd((1, 2, 11, 8), 104), rnd((1, 2, 27, 8), 105)
    v1, v2 = rnd((1, 2, 27, 8), 106), rnd((1, 2, 27, 8), 107)
    o1, l1 = oracle_mod.attn_fwd(q, k, v1, 0.4, causal=True)
    o2, _ = oracle_mod.attn_fwd(q, k, v2, 0.4, causal=True)
    o12, l12 = oracle_mod.attn_fwd(q, k, 2.0 * v1 - 3.0 * v2, 0.4, causal=True)
    np.testing.assert_allclose(o12, 2.0 * o1 - 3.0 * o2, atol=1e-12)
    np.testing.assert_array_equal(l12, l1)          # the scores do not depend on V


def test_common_key_shift_moves_each_row_uniformly(oracle_mod):
    q, k, v = rnd((1, 3, 9, 8), 108), rnd((1, 3, 21, 8), 109), rnd((1, 3, 21, 8), 110)
    c = rnd((8,), 111)
    scale = 0.25
    o, lse = oracle_mod.attn_fwd(q, k, v, scale)
    o2, lse2 = oracle_mod.attn_fwd(q, k + c, v, scale)
    np.testing.assert_allclose(o2, o, atol=1e-12)
    np.testing.assert_allclose(lse2, lse + scale * (q @ c), atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_backward_sums_over_keys(oracle_mod, causal):
    B, Hq, Hkv, Sq, Sk, D = 2, 6, 2, 13, 29, 8
    q, k, v = rnd((B, Hq, Sq, D), 112), rnd((B, Hkv, Sk, D), 113), rnd((B, Hkv, Sk, D), 114)
    do = rnd((B, Hq, Sq, D), 115)
    dq, dk, dv, _, _ = oracle_mod.attn_bwd(q, k, v, do, 0.35, causal=causal)
    G = Hq // Hkv
    # rows of dS sum to zero: dK summed over keys vanishes for every head dim
    np.testing.assert_allclose(dk.sum(axis=2), 0.0, atol=1e-11)
    # rows of P sum to one: dV summed over keys = dO summed over the group's rows
    # (every query row sees at least one key here)
    want = do.reshape(B, Hkv, G, Sq, D).sum(axis=(2, 3))
    np.testing.assert_allclose(dv.sum(axis=2), want, atol=1e-11)
    assert np.abs(dq).max() > 1e-3                  # not trivially zero
