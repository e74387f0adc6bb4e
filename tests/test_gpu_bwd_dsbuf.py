"""GPU parity of the backward with dS stored (attn_bwd_dsbuf: the dK/dV pass
writes its bf16 dS tiles to the workspace, dQ is the product dS K read back)
against the CPU fp64 oracle, and its bitwise properties: repeat runs, batch
composition, head slicing.

Bars as for the other backward paths: per tensor, max abs <= 2e-2 *
max(1, max |ref|) and normalised RMS <= 1e-2.  dK and dV come from the same
kernel as attn_bwd's and agree with it bitwise; dQ agrees within tolerance
(its dS is formed from the transposed S).
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import grad_errors, grad_ok, np_bits
from workloads import Workload, make_bwd_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def fwd_bwd(h, x, causal):
    out, lse = h.attn_fwd(x["q"], x["k"], x["v"], causal=causal)
    dq, dk, dv = h.attn_bwd_dsbuf(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    assert h.get_device_error() == 0
    return out, lse, dq, dk, dv


def check(h, w):
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    out, lse, dq, dk, dv = fwd_bwd(h, x, w.causal)
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(*(np_bits(x_cpu[n]) for n in ("q", "k", "v", "dout")), w.scale,
                                          causal=w.causal)
    errs = {n: grad_errors(g, r) for n, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv))}
    for n, e in errs.items():
        assert grad_ok(e), (n, errs)
    # dK and dV: the dK/dV kernel of attn_bwd, bitwise
    _, dk2, dv2 = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=w.causal)
    assert torch.equal(dk.view(torch.int16), dk2.view(torch.int16))
    assert torch.equal(dv.view(torch.int16), dv2.view(torch.int16))
    return errs


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (1, 1, 1, 128, 128, False),
    (1, 2, 1, 77, 300, False),          # ragged query and key tails
    (2, 4, 2, 300, 300, True),
    (1, 2, 2, 129, 1100, True),         # causal, Sq < Sk
    (1, 4, 1, 513, 257, False),
    (1, 24, 3, 1000, 1000, True),
    (2, 12, 4, 1100, 700, False),
    (2, 16, 16, 1300, 1300, True),      # more units than SMs in both kernels
])
def test_dsbuf_ragged(h, B, Hq, Hkv, Sq, Sk, causal):
    check(h, Workload("ds", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, seed=950 + Sq + Sk, backward=True))


def test_dsbuf_llm_heads_one_row(h):
    check(h, workloads.get("llm_gqa", B=1))


def test_dsbuf_repeat_and_batch_composition_bitwise(h):
    w = workloads.get("llm_gqa")
    x2 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=2).items()}
    x4 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=4).items()}
    r2 = fwd_bwd(h, x2, True)
    r2b = fwd_bwd(h, x2, True)
    r4 = fwd_bwd(h, x4, True)
    for a, b, c in zip(r2[2:], r2b[2:], r4[2:]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(c[:2].view(torch.int16), a.view(torch.int16))


def test_dsbuf_head_slice_bitwise(h):
    w = workloads.get("llm_gqa", B=1)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w, B=1).items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    xs = {"q": x["q"][:, 8:16].contiguous(), "dout": x["dout"][:, 8:16].contiguous(),
          "k": x["k"][:, 2:4].contiguous(), "v": x["v"][:, 2:4].contiguous()}
    _, _, dqs, dks, dvs = fwd_bwd(h, xs, True)
    assert torch.equal(dqs.view(torch.int16), dq[:, 8:16].view(torch.int16))
    assert torch.equal(dks.view(torch.int16), dk[:, 2:4].view(torch.int16))
    assert torch.equal(dvs.view(torch.int16), dv[:, 2:4].view(torch.int16))


def test_dsbuf_agrees_with_attn_bwd(h):
    w = workloads.get("llm_gqa")
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out, lse, dq, dk, dv = fwd_bwd(h, x, True)
    dq2, _, _ = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    e = grad_errors(dq, dq2.double().cpu().numpy())
    assert grad_ok(e), e


def test_dsbuf_llm_config_sums_over_keys(h):
    # full size, by properties that hold at any size (see test_gpu_bwd.py);
    # dQ rows 0..127 of head 3 against the oracle run on those rows alone
    w = workloads.get("llm_gqa")
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    G = w.Hq // w.Hkv
    dk_err = dk.double().sum(dim=2).abs() / dk.double().abs().sum(dim=2)
    want = x["dout"].double().view(w.B, w.Hkv, G, w.Sq, w.D).sum(dim=(2, 3))
    dv_err = (dv.double().sum(dim=2) - want).abs() / dv.double().abs().sum(dim=2)
    assert dk_err.max().item() <= 1e-2 and dv_err.max().item() <= 1e-2
    b, hd, rows = 1, 3, slice(0, 128)
    kvh = hd // G
    one = {"q": x_cpu["q"][b:b + 1, hd:hd + 1, rows], "dout": x_cpu["dout"][b:b + 1, hd:hd + 1, rows],
           "k": x_cpu["k"][b:b + 1, kvh:kvh + 1], "v": x_cpu["v"][b:b + 1, kvh:kvh + 1]}
    # causal, bottom-right aligned: query row q sees keys 0..q (Sq = Sk), so
    # the first 128 rows see only the first 128 keys
    one["k"] = one["k"][:, :, :128]
    one["v"] = one["v"][:, :, :128]
    rdq, _, _, _, _ = oracle.attn_bwd(*(np_bits(one[n]) for n in ("q", "k", "v", "dout")), w.scale, causal=True)
    e = grad_errors(dq[b:b + 1, hd:hd + 1, rows], rdq)
    assert grad_ok(e), e


def test_dsbuf_single_key_closed_form(h):
    # Sk = 1: dQ = dK = 0 and dV = sum_i dO_i
    g = torch.Generator().manual_seed(14)
    q = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    do = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    out, lse = h.attn_fwd(q, k, v)
    dq, dk, dv = h.attn_bwd_dsbuf(q, k, v, out, lse, do)
    assert h.get_device_error() == 0
    assert dq.float().abs().max() < 1e-3 and dk.float().abs().max() < 1e-2
    ref = do.double().sum(dim=2)
    assert np.allclose(dv[:, :, 0].double().cpu().numpy(), ref.cpu().numpy(), atol=2e-2 * max(1, ref.abs().max().item()))


def test_dsbuf_padded_keys_with_huge_p_do_not_reach_dq(h):
    # 100 identical keys (one key tile with 28 padded rows) and queries whose
    # scores are all about -200: for the padded rows, exp(0 - LSE) overflows.
    # Those rows are stored as zeros, so dQ stays finite; with identical keys
    # dQ = scale * k * sum_j dS_j = 0 exactly (rows of dS sum to zero).
    g = torch.Generator().manual_seed(15)
    u = torch.ones(128)
    k = u.expand(1, 2, 100, 128).to(torch.bfloat16).cuda()
    v = torch.randn(1, 2, 100, 128, generator=g).to(torch.bfloat16).cuda()
    q = (-200.0 * (128 ** 0.5) / 128.0 * u).expand(1, 2, 150, 128).to(torch.bfloat16).cuda()
    do = torch.randn(1, 2, 150, 128, generator=g).to(torch.bfloat16).cuda()
    out, lse = h.attn_fwd(q, k, v)
    assert lse.max().item() < -150
    dq, dk, dv = h.attn_bwd_dsbuf(q, k, v, out, lse, do)
    assert h.get_device_error() == 0
    assert torch.isfinite(dq.float()).all() and torch.isfinite(dk.float()).all() and torch.isfinite(dv.float()).all()
    assert dq.float().abs().max().item() < 1e-2
    dq2, _, _ = h.attn_bwd(q, k, v, out, lse, do)
    assert (dq.float() - dq2.float()).abs().max().item() < 1e-2


def test_dsbuf_many_heads_tiny_tiles(h):
    # B*Hq = 65600 query heads of 5 queries against 7 keys: 65600 one-tile
    # units in both kernels, every stored tile mostly padding (zeros past Sk,
    # zero P past Sq); rows agree bitwise with the same rows run alone and one
    # row with the oracle
    w = Workload("manyheads_ds", B=4100, Hq=16, Hkv=8, Sq=5, Sk=7, causal=False, seed=74)
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, False)
    for rows in (slice(0, 2), slice(4098, 4100)):
        xs = {k: v[rows].contiguous() for k, v in x.items()}
        _, _, dqs, dks, dvs = fwd_bwd(h, xs, False)
        for a, b in ((dqs, dq[rows]), (dks, dk[rows]), (dvs, dv[rows])):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    b = 4099
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(*(np_bits(x_cpu[n][b:b + 1]) for n in ("q", "k", "v", "dout")), w.scale)
    for n, g, r in (("dq", dq[b:b + 1], rdq), ("dk", dk[b:b + 1], rdk), ("dv", dv[b:b + 1], rdv)):
        e = grad_errors(g, r)
        assert grad_ok(e), (n, e)
