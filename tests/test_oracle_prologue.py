"""Pins of the oracle's e4m3 quantisation prologue (oracle/attn_oracle.c,
oracle_quantize_e4m3 and oracle_e4m3_rne) against things other than itself:
torch's own float8_e4m3fn cast, the e4m3fn value table, closed forms of the
RMS normalisation on special rows (restated in Python doubles), exact scale
invariance, and the harness's independent torch quantiser."""
import math

import numpy as np
import pytest
import torch

import oracle
from parity import check_e4m3_codes
from workloads import bf16_bits
from workloads.gen import quantize_e4m3_per_head


def torch_e4m3(v: torch.Tensor) -> np.ndarray:
    return v.float().clamp(-448, 448).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_rne_matches_torch_cast_across_magnitudes():
    g = torch.Generator().manual_seed(5)
    parts = [torch.randn(20000, generator=g) * s for s in (1e-3, 0.02, 1.0, 30.0, 300.0)]
    # exact ties: midpoints between neighbouring codes (normal and subnormal ranges)
    vals = torch.arange(0, 0x7E, dtype=torch.int32).to(torch.uint8).view(torch.float8_e4m3fn).float()
    mids = (vals[:-1] + vals[1:]) / 2
    v = torch.cat(parts + [mids, -mids, torch.tensor([0.0, -0.0, 448.0, 449.0, 1e6, -1e6, 2.0 ** -10, 2.0 ** -11])])
    ours = np.array([oracle.e4m3_rne(float(x)) for x in v.numpy()], dtype=np.uint8)
    assert np.array_equal(ours, torch_e4m3(v))


def test_rne_known_codes():
    # OCP e4m3fn: 1.0 = 0x38, 448 = 0x7E (largest finite), 2^-6 = 0x08 (smallest normal),
    # 2^-9 = 0x01 (smallest subnormal), 1.125 = 0x39; ties go to the even code
    assert oracle.e4m3_rne(1.0) == 0x38
    assert oracle.e4m3_rne(448.0) == 0x7E and oracle.e4m3_rne(1e9) == 0x7E and oracle.e4m3_rne(-1e9) == 0xFE
    assert oracle.e4m3_rne(2.0 ** -6) == 0x08 and oracle.e4m3_rne(2.0 ** -9) == 0x01
    assert oracle.e4m3_rne(1.125) == 0x39
    assert oracle.e4m3_rne(1.0625) == 0x38            # halfway 1.0 / 1.125 -> even code 0x38
    assert oracle.e4m3_rne(1.1875) == 0x3A            # halfway 1.125 / 1.25 -> even code 0x3A
    assert oracle.e4m3_rne(2.0 ** -10) == 0x00        # halfway 0 / 2^-9 -> 0
    assert oracle.e4m3_rne(-2.0 ** -12) == 0x80       # underflow keeps the sign


def _bits(x: torch.Tensor) -> np.ndarray:
    return bf16_bits(x.to(torch.bfloat16))


def test_plain_quantiser_matches_the_torch_harness():
    # without normalisation the definition is the harness's (independent torch
    # code); torch rounds the quotient to fp32 before its e4m3 cast, so a code
    # may differ where the exact quotient is within 2^-24 of a rounding midpoint
    g = torch.Generator().manual_seed(6)
    x = (torch.randn(2, 3, 100, 128, generator=g) * 2.5).to(torch.bfloat16)
    codes, ds, quot = oracle.quantize_e4m3(_bits(x), rmsnorm=False, with_quotient=True)
    ref_codes, ref_ds = quantize_e4m3_per_head(x)
    assert np.array_equal(ds, ref_ds.numpy())
    check_e4m3_codes(ref_codes.view(torch.uint8).numpy(), ref_ds.numpy(), codes, ds, quot,
                     descale_rel=0.0, boundary_rel=2.0 ** -23)


def test_quotients_are_the_definition():
    # the quotient the codes round is y / descale with y = x (no norm) or
    # x / sqrt(mean x^2 + eps), in doubles
    g = torch.Generator().manual_seed(16)
    x = (torch.randn(1, 2, 9, 128, generator=g) * 0.7).to(torch.bfloat16)
    xd = x.double().numpy()
    for rms in (False, True):
        codes, ds, quot = oracle.quantize_e4m3(_bits(x), rmsnorm=rms, eps=1e-6, with_quotient=True)
        y = xd / np.sqrt((xd * xd).mean(axis=-1, keepdims=True) + 1e-6) if rms else xd
        np.testing.assert_allclose(quot, y / ds.astype(np.float64)[:, :, None, None], rtol=1e-14, atol=0)
        for h in range(2):
            assert ds[0, h] == np.float32(np.abs(y[0, h]).max() / 448.0)


def test_single_nonzero_element_takes_the_largest_code():
    x = torch.zeros(1, 2, 7, 128)
    x[0, 0, 3, 17] = -3.5
    x[0, 1, 6, 127] = 0.25
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=False)
    assert ds[0, 0] == np.float32(3.5) / np.float32(448) and ds[0, 1] == np.float32(0.25) / np.float32(448)
    assert codes[0, 0, 3, 17] == 0xFE and codes[0, 1, 6, 127] == 0x7E
    mask = np.ones(codes.shape, bool)
    mask[0, 0, 3, 17] = mask[0, 1, 6, 127] = False
    assert np.all(codes[mask] == 0)


def test_all_zero_head_has_unit_descale():
    x = torch.zeros(1, 1, 5, 128)
    for rms in (False, True):
        codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=rms)
        assert ds[0, 0] == 1.0 and np.all(codes == 0)


def _factor(ss, eps):
    """r = 1 / sqrt(ss / 128 + eps) in doubles."""
    return 1.0 / math.sqrt(ss / 128.0 + eps)


def test_rmsnorm_closed_form_one_spike_per_row():
    # a row whose only nonzero value is a has y = a / sqrt(a^2 / 128 + eps) there
    a_vals = [0.5, -1.0, 2.0, 3.0, -0.75, 1.5]
    x = torch.zeros(1, 1, len(a_vals), 128)
    for i, a in enumerate(a_vals):
        x[0, 0, i, (7 * i) % 128] = a
    eps = 1e-6
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=True, eps=eps)
    y = [a * _factor(a * a, eps) for a in a_vals]
    amax = max(abs(v) for v in y)
    assert ds[0, 0] == np.float32(amax / 448.0)
    for i, v in enumerate(y):
        assert codes[0, 0, i, (7 * i) % 128] == oracle.e4m3_rne(v / float(ds[0, 0]))
    mask = np.ones(codes.shape, bool)
    for i in range(len(a_vals)):
        mask[0, 0, i, (7 * i) % 128] = False
    assert np.all(codes[mask] == 0)


def test_rmsnorm_closed_form_constant_rows():
    # a constant row a has y = a / sqrt(a^2 + eps) everywhere: all of a head's
    # rows with the same |a| take the largest code
    x = torch.full((1, 2, 4, 128), 0.75)
    x[0, 1] = -2.0
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=True, eps=1e-6)
    assert ds[0, 0] == np.float32(0.75 / math.sqrt(0.75 ** 2 + 1e-6) / 448.0)
    assert ds[0, 1] == np.float32(2.0 / math.sqrt(4.0 + 1e-6) / 448.0)
    assert np.all(codes[0, 0] == 0x7E) and np.all(codes[0, 1] == 0xFE)


def test_rmsnorm_closed_form_sums():
    # rows with known sums of squares: distinct powers of two, 1 + 16, and 128 / 4
    x = torch.zeros(1, 1, 3, 128)
    for d in range(0, 128, 8):
        x[0, 0, 0, d] = 2.0 ** (d // 8 - 8)            # squares 2^-16 .. 2^14, each once
    x[0, 0, 1, 5] = 1.0
    x[0, 0, 1, 77] = -4.0                              # 1 + 16
    x[0, 0, 2, :] = torch.tensor([(-1.0) ** d * 0.5 for d in range(128)])   # 128 / 4
    sums = [sum(4.0 ** (k - 8) for k in range(16)), 17.0, 32.0]
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=True, eps=1e-6)
    ys = [x[0, 0, i].double().numpy() * _factor(sums[i], 1e-6) for i in range(3)]
    amax = max(float(np.abs(y).max()) for y in ys)
    assert ds[0, 0] == np.float32(amax / 448.0)
    for i in range(3):
        want = [oracle.e4m3_rne(float(v) / float(ds[0, 0])) for v in ys[i]]
        assert list(codes[0, 0, i]) == want


def test_rmsnorm_half_row_sum():
    # the sum runs over all 128 values: a row that is a in the first half and b
    # in the second has mean (a^2 + b^2) / 2
    x = torch.zeros(1, 1, 2, 128)
    x[0, 0, 0, :64] = 1.0
    x[0, 0, 0, 64:] = 3.0
    x[0, 0, 1, :] = 1.0
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=True, eps=1e-6)
    y_hi = 3.0 / math.sqrt(5.0 + 1e-6)
    assert ds[0, 0] == np.float32(y_hi / 448.0)
    assert codes[0, 0, 0, 100] == 0x7E
    assert codes[0, 0, 0, 10] == oracle.e4m3_rne(1.0 / math.sqrt(5.0 + 1e-6) / float(ds[0, 0]))
    assert codes[0, 0, 1, 10] == oracle.e4m3_rne(1.0 / math.sqrt(1.0 + 1e-6) / float(ds[0, 0]))


def test_rmsnorm_removes_power_of_two_scales_exactly():
    # with eps = 0 the normalised values of 2^k x equal those of x bit for bit
    g = torch.Generator().manual_seed(7)
    x = torch.randn(1, 2, 33, 128, generator=g).to(torch.bfloat16)
    c0, d0 = oracle.quantize_e4m3(_bits(x), rmsnorm=True, eps=0.0)
    for k in (-3, 5):
        c1, d1 = oracle.quantize_e4m3(_bits(x.float() * 2.0 ** k), rmsnorm=True, eps=0.0)
        assert np.array_equal(c0, c1) and np.array_equal(d0, d1)


def test_dequantised_error_within_half_a_code_step():
    g = torch.Generator().manual_seed(8)
    x = torch.randn(1, 1, 64, 128, generator=g).to(torch.bfloat16)
    codes, ds = oracle.quantize_e4m3(_bits(x), rmsnorm=False)
    y = x.float().numpy()[0, 0]
    q = y / ds[0, 0]
    deq = np.vectorize(oracle.e4m3_to_double)(codes[0, 0]).astype(np.float64)
    # code step at |q|: 2^(floor(log2|q|) - 3) in the normal range, 2^-9 below 2^-6
    e = np.floor(np.log2(np.maximum(np.abs(q), 2.0 ** -6)))
    step = np.exp2(e - 3)
    assert np.all(np.abs(deq - q) <= step / 2 + 1e-12)
