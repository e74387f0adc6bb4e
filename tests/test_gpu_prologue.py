"""GPU parity of the e4m3 quantisation prologue (attn_quantize_e4m3) against the
oracle, at small ragged shapes and on the full Q of the fp8 config: the kernel
normalises in fp32, the oracle in fp64, so descales agree within a relative
2^-17 and codes agree except next to an e4m3 rounding midpoint (within a
relative 2^-16 of the oracle's quotient), where they differ by one step (the
rule and its derivation are in tests/parity.py); without normalisation the
descales are bit-equal.  Also invariance under head slicing, and the whole
fp8 pipeline (product prologue, then attn_fwd) against the oracle on the
dequantized values."""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import FP8_NRMS, check_e4m3_codes, fwd_errors, oracle_fwd
from workloads import Workload, bf16_bits, make_fwd_inputs, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def check_exact(h, x, rmsnorm, eps=1e-6, max_frac=1e-3):
    """Prologue on the GPU against the oracle under the e4m3 parity rule; the
    number of codes that differ (each next to a rounding boundary) is reported
    and bounded: by max_frac of the elements with the norm, by zero without it
    (y = x exactly, and both sides round the exact quotient).  With the norm
    the bound is loose for heads of few rows: in the row of a head's largest
    value, 448 x / x_max is often exactly an e4m3 midpoint, and which side the
    fp32 and fp64 values of y fall on is then a matter of their rounding."""
    codes, ds = h.quantize_e4m3(x.cuda(), rmsnorm=rmsnorm, eps=eps)
    assert h.get_device_error() == 0
    ref_codes, ref_ds, quot = oracle.quantize_e4m3(bf16_bits(x), rmsnorm=rmsnorm, eps=eps, with_quotient=True)
    got_ds = ds.cpu().numpy()
    if not rmsnorm:
        # y = x exactly: both sides round amax / 448 once to fp32
        assert np.array_equal(got_ds.view(np.uint32), ref_ds.view(np.uint32))
    n_diff = check_e4m3_codes(codes.view(torch.uint8).cpu().numpy(), got_ds, ref_codes, ref_ds, quot)
    print("e4m3 codes differing next to a rounding boundary: %d of %d" % (n_diff, ref_codes.size))
    assert n_diff <= (max_frac * ref_codes.size if rmsnorm else 0), n_diff
    return codes, ds


@pytest.mark.parametrize("B,H,S", [(1, 1, 1), (1, 3, 37), (2, 2, 300), (1, 4, 1000), (3, 1, 257)])
@pytest.mark.parametrize("rmsnorm", [False, True])
def test_prologue_small(h, B, H, S, rmsnorm):
    g = torch.Generator().manual_seed(1000 + S + B)
    x = (torch.randn(B, H, S, 128, generator=g) * 1.7).to(torch.bfloat16)
    check_exact(h, x, rmsnorm)


def test_prologue_special_rows(h):
    x = torch.zeros(1, 3, 40, 128)
    x[0, 0, 5, 9] = -3.5                            # one spike: the largest code
    x[0, 1] = 0.75                                  # constant rows
    x[0, 2, :, :] = torch.linspace(-1e-3, 1e-3, 40 * 128).view(40, 128)   # small values, subnormal codes
    for rms in (False, True):
        check_exact(h, x.to(torch.bfloat16), rms)
    check_exact(h, torch.zeros(1, 1, 9, 128, dtype=torch.bfloat16), True)   # all-zero head: descale 1


def test_prologue_extreme_magnitudes(h):
    # squares that underflow to fp32 subnormals (2^-70 scale), large rows (2^60),
    # a mix inside one row, and a head whose descale is tiny: every fp32 step of
    # the norm and of the quotient is IEEE on both sides
    g = torch.Generator().manual_seed(31)
    x = torch.randn(1, 3, 48, 128, generator=g)
    x[0, 0, :16] *= 2.0 ** -70
    x[0, 0, 16:32] *= 2.0 ** 60
    x[0, 1, :, ::3] *= 2.0 ** -64
    x[0, 2] *= 2.0 ** -80                           # a whole head of tiny values: tiny descale
    for rms in (False, True):
        check_exact(h, x.to(torch.bfloat16), rms)


def test_prologue_more_than_65535_heads(h):
    # 70000 heads: more than a grid's y dimension holds, so CTAs stride over heads
    g = torch.Generator().manual_seed(33)
    x = (torch.randn(2, 35000, 3, 128, generator=g) * 1.3).to(torch.bfloat16)
    check_exact(h, x, True)
    check_exact(h, x, False)


def test_prologue_fp8_config_q(h):
    w = workloads.get("fp8")
    g = torch.Generator().manual_seed(w.seed)
    x = torch.randn(w.B, w.Hq, w.Sq, w.D, generator=g).to(torch.bfloat16)
    check_exact(h, x, True, max_frac=1e-5)
    check_exact(h, x, False)


def test_prologue_head_slice_bitwise(h):
    g = torch.Generator().manual_seed(12)
    x = torch.randn(2, 6, 500, 128, generator=g).to(torch.bfloat16).cuda()
    c, d = h.quantize_e4m3(x, rmsnorm=True)
    cs, ds = h.quantize_e4m3(x[1:, 2:5].contiguous(), rmsnorm=True)
    assert torch.equal(cs.view(torch.uint8), c[1:, 2:5].view(torch.uint8)) and torch.equal(ds, d[1:, 2:5])


def test_fp8_pipeline_prologue_then_attention(h):
    # product path end to end: bf16 Q/K/V -> prologue (Q/K normalised) -> e4m3 attention
    w = Workload("pipe", B=1, Hq=4, Hkv=2, Sq=700, Sk=900, seed=21)
    x = make_fwd_inputs(w)
    qc, qd = h.quantize_e4m3(x["q"].cuda(), rmsnorm=True)
    kc, kd = h.quantize_e4m3(x["k"].cuda(), rmsnorm=True)
    vc, vd = h.quantize_e4m3(x["v"].cuda(), rmsnorm=False)
    out, lse = h.attn_fwd(qc, kc, vc, q_descale=qd, k_descale=kd, v_descale=vd)
    assert h.get_device_error() == 0
    o_ref, lse_ref = oracle_fwd(qc.cpu(), kc.cpu(), vc.cpu(), w.scale, False, descales=(qd, kd, vd))
    e = fwd_errors(out, lse, o_ref, lse_ref, None)
    assert e["o_nrms"] <= FP8_NRMS, e
