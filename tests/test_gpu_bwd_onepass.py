"""GPU parity of the one-pass backward (attn_bwd_onepass: dQ, dK, dV from one
kernel, dQ added in ascending key-tile order) against the CPU fp64 oracle,
and its bitwise properties: repeat runs, batch composition, head slicing.

Bars as for the two-kernel backward: per tensor, max abs <= 2e-2 *
max(1, max |ref|) and normalised RMS <= 1e-2.  The two backward paths sum in
different fixed orders, so they agree within that tolerance, not bitwise.
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
    dq, dk, dv = h.attn_bwd_onepass(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
    assert h.get_device_error() == 0
    return out, lse, dq, dk, dv


def check(h, w):
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, w.causal)
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(*(np_bits(x_cpu[n]) for n in ("q", "k", "v", "dout")), w.scale,
                                          causal=w.causal)
    errs = {n: grad_errors(g, r) for n, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv))}
    for n, e in errs.items():
        assert grad_ok(e), (n, errs)
    return errs


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (1, 1, 1, 128, 128, False),         # one tile pair: key tile 0 is also the last contributor
    (1, 2, 1, 77, 300, False),
    (2, 4, 2, 300, 300, True),
    (1, 2, 2, 129, 1100, True),         # causal, Sq < Sk: early key tiles see every query
    (1, 4, 1, 513, 257, False),
    (1, 24, 3, 1000, 1000, True),
    (2, 12, 4, 1100, 700, False),
    # more key-tile units than SMs: each CTA takes several units, and the
    # ordered dQ additions run across units dealt to different CTAs
    (2, 16, 16, 1300, 1300, True),
    (1, 40, 20, 900, 1000, True),
])
def test_onepass_ragged(h, B, Hq, Hkv, Sq, Sk, causal):
    check(h, Workload("op", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, seed=900 + Sq + Sk, backward=True))


def test_onepass_llm_heads_one_row(h):
    # Qwen3-8B head layout (Hq=32, Hkv=8) at S=2048, causal, one batch row
    check(h, workloads.get("llm_gqa", B=1))


def test_onepass_repeat_and_batch_composition_bitwise(h):
    w = workloads.get("llm_gqa")
    x2 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=2).items()}
    x4 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=4).items()}
    r2 = fwd_bwd(h, x2, True)
    r2b = fwd_bwd(h, x2, True)
    r4 = fwd_bwd(h, x4, True)
    for a, b, c in zip(r2[2:], r2b[2:], r4[2:]):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
        assert torch.equal(c[:2].view(torch.int16), a.view(torch.int16))


def test_onepass_head_slice_bitwise(h):
    w = workloads.get("llm_gqa", B=1)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w, B=1).items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    xs = {"q": x["q"][:, 8:16].contiguous(), "dout": x["dout"][:, 8:16].contiguous(),
          "k": x["k"][:, 2:4].contiguous(), "v": x["v"][:, 2:4].contiguous()}
    _, _, dqs, dks, dvs = fwd_bwd(h, xs, True)
    assert torch.equal(dqs.view(torch.int16), dq[:, 8:16].view(torch.int16))
    assert torch.equal(dks.view(torch.int16), dk[:, 2:4].view(torch.int16))
    assert torch.equal(dvs.view(torch.int16), dv[:, 2:4].view(torch.int16))


def test_onepass_agrees_with_two_kernel_backward(h):
    w = workloads.get("llm_gqa")
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out, lse, dq, dk, dv = fwd_bwd(h, x, True)
    dq2, dk2, dv2 = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    for n, a, b in (("dq", dq, dq2), ("dk", dk, dk2), ("dv", dv, dv2)):
        e = grad_errors(a, b.double().cpu().numpy())
        assert grad_ok(e), (n, e)


def test_onepass_single_key_closed_form(h):
    # Sk = 1: dQ = dK = 0 and dV = sum_i dO_i
    g = torch.Generator().manual_seed(13)
    q = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    do = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    out, lse = h.attn_fwd(q, k, v)
    dq, dk, dv = h.attn_bwd_onepass(q, k, v, out, lse, do)
    assert h.get_device_error() == 0
    assert dq.float().abs().max() < 1e-3 and dk.float().abs().max() < 1e-2
    ref = do.double().sum(dim=2)
    assert np.allclose(dv[:, :, 0].double().cpu().numpy(), ref.cpu().numpy(), atol=2e-2 * max(1, ref.abs().max().item()))


def test_onepass_llm_config_sums_over_keys(h):
    # the bench's backward config at full size, by properties that hold at any
    # size (see test_gpu_bwd.py): dK summed over keys vanishes, dV summed over
    # keys equals the group's dO summed over rows
    w = workloads.get("llm_gqa")
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    G = w.Hq // w.Hkv
    dk_err = dk.double().sum(dim=2).abs() / dk.double().abs().sum(dim=2)
    want = x["dout"].double().view(w.B, w.Hkv, G, w.Sq, w.D).sum(dim=(2, 3))
    dv_err = (dv.double().sum(dim=2) - want).abs() / dv.double().abs().sum(dim=2)
    assert dk_err.max().item() <= 1e-2 and dv_err.max().item() <= 1e-2


def test_onepass_many_heads_and_rows(h):
    # B*Hq = 65600 query heads of one query tile each: 32800 key-tile units,
    # every dQ tile from a single contributor; rows agree bitwise with the
    # same rows run alone, and one row with the oracle
    w = Workload("manyheads_op", B=4100, Hq=16, Hkv=8, Sq=5, Sk=7, causal=False, seed=72)
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, False)
    for rows in (slice(0, 2), slice(4098, 4100)):
        xs = {k: v[rows].contiguous() for k, v in x.items()}
        _, _, dqs, dks, dvs = fwd_bwd(h, xs, False)
        assert torch.equal(dqs.view(torch.int16), dq[rows].view(torch.int16))
        assert torch.equal(dks.view(torch.int16), dk[rows].view(torch.int16))
        assert torch.equal(dvs.view(torch.int16), dv[rows].view(torch.int16))
    b = 4099
    rdq, rdk, rdv, _, _ = oracle.attn_bwd(*(np_bits(x_cpu[n][b:b + 1]) for n in ("q", "k", "v", "dout")), w.scale)
    for n, g, r in (("dq", dq[b:b + 1], rdq), ("dk", dk[b:b + 1], rdk), ("dv", dv[b:b + 1], rdv)):
        e = grad_errors(g, r)
        assert grad_ok(e), (n, e)


def test_onepass_long_sequence_many_contributors(h):
    # 64 key tiles add into every dQ tile (non-causal S8192, one head pair):
    # long ordered chains, compared with the two-kernel backward
    w = Workload("long_op", B=1, Hq=2, Hkv=1, Sq=8192, Sk=8192, causal=False, seed=73)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out, lse, dq, dk, dv = fwd_bwd(h, x, False)
    dq2, dk2, dv2 = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"])
    for n, a, b in (("dq", dq, dq2), ("dk", dk, dk2), ("dv", dv, dv2)):
        e = grad_errors(a, b.double().cpu().numpy())
        assert grad_ok(e), (n, e)
