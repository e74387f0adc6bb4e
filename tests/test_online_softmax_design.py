"""The forward kernel's softmax recurrence, restated on the CPU in fp64, against
the oracle: base-2 online softmax over 128-key tiles with a lazy rescale (the
running maximum m used for the exponentials moves only when a tile's maximum
exceeds it by more than 8 in log2 units), so that O and l always share the
same stale maximum and O / l is the softmax average exactly, whatever the
rescale schedule.  Checks the two facts the kernel relies on: the result
equals the plain definition, and every probability the kernel forms before
rounding it to 16 bits stays at most 2^8 (well inside fp16 and bf16).

This is a statement of the algorithm, not of the kernel's code; it shares
nothing with either side of the parity tests.
"""
import math

import numpy as np
import pytest

import oracle

TILE = 128
THRESHOLD = 8.0


def online_softmax_rows(s2, v, lazy):
    """Rows of O = softmax(s) V with s2 = s * log2(e), folded tile by tile.
    Returns (O, LSE in natural log, largest probability formed)."""
    n, sk = s2.shape
    m = np.full(n, -np.inf)
    l = np.zeros(n)
    o = np.zeros((n, v.shape[1]))
    p_max = 0.0
    for t0 in range(0, sk, TILE):
        st = s2[:, t0:t0 + TILE]
        m_tile = st.max(axis=1)
        rise = m_tile - m
        move = rise > (THRESHOLD if lazy else 0.0)
        m_new = np.where(move, m_tile, m)
        corr = np.where(np.isfinite(m), np.exp2(m - m_new), 0.0)
        o *= corr[:, None]
        l *= corr
        p = np.exp2(st - m_new[:, None])
        p_max = max(p_max, float(p.max()))
        l += p.sum(axis=1)
        o += p @ v[t0:t0 + TILE]
        m = m_new
    return o / l[:, None], (m + np.log2(l)) * math.log(2.0), p_max


@pytest.mark.parametrize("slope", [0.0, 3.0, 20.0, -15.0])
def test_lazy_rescale_is_exact_and_bounds_p(slope):
    rng = np.random.default_rng(int(slope * 10) + 1000)
    sq, sk, d = 40, 777, 16
    q = rng.standard_normal((1, 1, sq, d))
    k = rng.standard_normal((1, 1, sk, d))
    v = rng.standard_normal((1, 1, sk, d))
    # a per-key ramp through the last dimension (q_d = 1, k_d = ramp): scores
    # rise by `slope` (log2 units) per tile on top of the random part
    q[..., -1] = 1.0
    k[0, 0, :, -1] = np.arange(sk) * (slope / TILE) / math.log2(math.e)
    o_ref, lse_ref = oracle.attn_fwd(q, k, v, 1.0)
    s2 = (q[0, 0] @ k[0, 0].T) * math.log2(math.e)
    for lazy in (False, True):
        o, lse, p_max = online_softmax_rows(s2, v[0, 0], lazy)
        np.testing.assert_allclose(o, o_ref[0, 0], rtol=0, atol=1e-12)
        np.testing.assert_allclose(lse, lse_ref[0, 0], rtol=0, atol=1e-11)
        assert p_max <= (2.0 ** THRESHOLD if lazy else 1.0) * (1 + 1e-12)
        if lazy and slope == 3.0:
            assert p_max > 4.0          # the stale maximum was really kept over tiles
