"""Facts the e4m3 prologue kernel relies on, restated on the CPU.

The e4m3 midpoint test (e4m3_midpoint in csrc/prep_kernel.cuh) recognises an
fp32 value lying exactly on a rounding boundary of e4m3fn from its bits; the
same bit rule is written out here and checked against the midpoints of the
value table torch's float8 type decodes, and against brute force on values
next to them.

The head maximum: each CTA stores the
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


def midpoint_by_bits(q):
    """The kernel's bit rule for 'q is exactly an e4m3 rounding midpoint'."""
    u = int(bits(np.float32(q))) & 0x7FFFFFFF
    e = (u >> 23) - 127
    if e > 8 or e < -10:
        return False
    if e == -10:
        return u == (117 << 23)
    half = (1 << 19) if e >= -6 else (1 << (13 - e))
    return (u & ((half << 1) - 1)) == half


def test_midpoint_bit_rule_matches_the_value_table():
    import torch

    vals = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    mids = set(float(m) for m in (vals[:-1] + vals[1:]) / 2)
    mids.add(464.0)                   # between 448 and the first value past the range: saturates either way
    for m in mids:
        assert midpoint_by_bits(m) and midpoint_by_bits(-m), m
        for nb in (np.nextafter(np.float32(m), np.float32(0)), np.nextafter(np.float32(m), np.float32(1e9))):
            assert not midpoint_by_bits(nb), (m, nb)
    rng = np.random.default_rng(5)
    for q in np.ldexp(rng.random(20000).astype(np.float32) + np.float32(0.5), rng.integers(-14, 10, 20000)):
        q = np.float32(q)
        assert midpoint_by_bits(q) == (float(abs(q)) in mids), q
    for q in (0.0, 2.0 ** -11, 2.0 ** -9, 448.0, 512.0, 1e30):
        assert not midpoint_by_bits(q), q
