"""The e4m3 prologue's head maximum, restated on the CPU: each CTA stores the
negated maximum of its rows into a zeroed 32-bit slot with an unsigned
atomicMax on the float's bit pattern.  That is order-independent only if the
bit patterns of non-positive floats order like unsigned integers by
magnitude, with every negative value above the zeroed slot, and a finished
descale (a positive float) must be told apart from a pending maximum by its
sign bit.  These are facts of the IEEE-754 binary32 encoding, checked here
exhaustively over exponents and on random mantissas.
"""
import numpy as np


def bits(x):
    return np.asarray(x, dtype=np.float32).view(np.uint32)


def test_negated_magnitudes_order_like_unsigned_integers():
    rng = np.random.default_rng(3)
    mags = np.concatenate([
        np.float32([0.0, 1e-45, 1.17549435e-38, 1.0, 3.4028235e38]),
        np.ldexp(np.float32(1.0) + rng.random(4000, dtype=np.float32), rng.integers(-149, 127, 4000)).astype(np.float32),
    ])
    mags = mags[np.isfinite(mags)]
    neg = bits(-mags)
    order_by_bits = np.argsort(neg, kind="stable")
    order_by_mag = np.argsort(mags, kind="stable")
    np.testing.assert_array_equal(mags[order_by_bits], mags[order_by_mag])


def test_every_pending_maximum_beats_the_zeroed_slot_and_keeps_its_sign():
    # -0.0 (an all-zero head) and every negative value are above the memset 0 slot
    assert bits(np.float32(-0.0)) > bits(np.float32(0.0))
    assert bits(np.float32(-1e-45)) > bits(np.float32(-0.0))
    # a descale is positive: sign bit clear, so it is never read as a pending maximum
    for ds in (np.float32(1.0), np.float32(1e-30), np.float32(448.0) / np.float32(448.0)):
        assert (bits(ds) >> 31) == 0
    assert (bits(np.float32(-0.0)) >> 31) == 1
