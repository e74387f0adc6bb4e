"""GPU parity of the deterministic backward against the CPU fp64 oracle, and
its bitwise properties (repeat runs, batch composition, head slicing).

Bar (the pages give none for gradients): for each of dQ, dK, dV,
max abs <= 2e-2 * max(1, max |ref|) and normalised RMS <= 1e-2.
"""
import math

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
    dq, dk, dv = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=causal)
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
    (1, 1, 1, 128, 128, False),
    (1, 2, 1, 77, 300, False),
    (2, 4, 2, 300, 300, True),
    (1, 2, 2, 129, 1100, True),
    (1, 4, 1, 513, 257, False),
    # more query-tile units than SMs, ragged tails: the persistent dQ CTAs each
    # take several units of different lengths
    (1, 24, 3, 1000, 1000, True),
    (2, 12, 4, 1100, 700, False),
    # more key-tile units than SMs: the persistent dK/dV CTAs take several
    # (352 and 160 units, causal, ragged tails, grouped heads)
    (2, 16, 16, 1300, 1300, True),
    (1, 40, 20, 900, 1000, True),
])
def test_bwd_ragged(h, B, Hq, Hkv, Sq, Sk, causal):
    check(h, Workload("bw", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, seed=200 + Sq + Sk, backward=True))


def test_bwd_llm_heads_one_row(h):
    # Qwen3-8B head layout (Hq=32, Hkv=8) at S=2048, causal, one batch row
    check(h, workloads.get("llm_gqa", B=1))


def test_bwd_repeat_and_batch_composition_bitwise(h):
    w = workloads.get("llm_gqa")
    x2 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=2).items()}
    x4 = {k: v.cuda() for k, v in make_bwd_inputs(w, B=4).items()}
    r2 = fwd_bwd(h, x2, True)
    r2b = fwd_bwd(h, x2, True)
    r4 = fwd_bwd(h, x4, True)
    for a, b, c in zip(r2, r2b, r4):
        ai = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32)
        bi = b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)
        ci = c.view(torch.int16) if c.dtype == torch.bfloat16 else c.view(torch.int32)
        assert torch.equal(ai, bi)
        assert torch.equal(ci[:2], ai)


def test_bwd_head_slice_bitwise(h):
    w = workloads.get("llm_gqa", B=1)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w, B=1).items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    xs = {"q": x["q"][:, 8:16].contiguous(), "dout": x["dout"][:, 8:16].contiguous(),
          "k": x["k"][:, 2:4].contiguous(), "v": x["v"][:, 2:4].contiguous()}
    _, _, dqs, dks, dvs = fwd_bwd(h, xs, True)
    assert torch.equal(dqs.view(torch.int16), dq[:, 8:16].view(torch.int16))
    assert torch.equal(dks.view(torch.int16), dk[:, 2:4].view(torch.int16))
    assert torch.equal(dvs.view(torch.int16), dv[:, 2:4].view(torch.int16))


def test_bwd_single_key_closed_form(h):
    # Sk = 1: dQ = dK = 0 and dV = sum_i dO_i
    g = torch.Generator().manual_seed(12)
    q = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    k = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    v = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16).cuda()
    do = torch.randn(1, 2, 200, 128, generator=g).to(torch.bfloat16).cuda()
    out, lse = h.attn_fwd(q, k, v)
    dq, dk, dv = h.attn_bwd(q, k, v, out, lse, do)
    assert h.get_device_error() == 0
    assert dq.float().abs().max() < 1e-3 and dk.float().abs().max() < 1e-2
    ref = do.double().sum(dim=2)
    assert np.allclose(dv[:, :, 0].double().cpu().numpy(), ref.cpu().numpy(), atol=2e-2 * max(1, ref.abs().max().item()))


def test_bwd_llm_config_sums_over_keys(h):
    # the bench's backward (B=2, Hq=32, Hkv=8, S=2048, causal) at full size,
    # checked by properties that hold at any size: rows of dS sum to zero, so
    # dK summed over keys vanishes; rows of P sum to one, so dV summed over
    # keys equals dO summed over the rows of the KV head's query heads.  With
    # bf16 P, dS and outputs the identities hold to a small fraction of each
    # sum's absolute mass; a wrong or missing term breaks them at order one.
    w = workloads.get("llm_gqa")
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    _, _, dq, dk, dv = fwd_bwd(h, x, True)
    G = w.Hq // w.Hkv
    dk_err = dk.double().sum(dim=2).abs() / dk.double().abs().sum(dim=2)
    want = x["dout"].double().view(w.B, w.Hkv, G, w.Sq, w.D).sum(dim=(2, 3))
    dv_err = (dv.double().sum(dim=2) - want).abs() / dv.double().abs().sum(dim=2)
    print("max relative sums: dK %.3e, dV %.3e" % (dk_err.max().item(), dv_err.max().item()))
    assert dk_err.max().item() <= 1e-2 and dv_err.max().item() <= 1e-2


def test_bwd_more_than_65535_heads(h):
    # B*Hq = 65600 query heads (more than a grid's y dimension holds): rows of
    # the batch agree bit for bit with the same rows run alone, and one row
    # with the oracle
    w = Workload("manyheads", B=4100, Hq=16, Hkv=8, Sq=5, Sk=7, causal=False, seed=71)
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


@pytest.mark.parametrize("causal", [True, False])
def test_back_to_back_calls_on_one_stream(h, causal):
    # Forward and backward calls queued on one stream with no host sync,
    # reusing the same output buffers and workspace: each grid waits for the
    # grid before it before touching memory (the dQ grid also for dK/dV before
    # it exits), so after the queue drains the buffers hold bitwise the last
    # calls' results, as when those calls run alone.
    w = Workload("b2b", B=1, Hq=8, Hkv=2, Sq=1000, Sk=1000, causal=causal, seed=90)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    g = torch.Generator().manual_seed(91)
    q2 = torch.randn(x["q"].shape, generator=g).to(torch.bfloat16).cuda()
    do2 = torch.randn(x["dout"].shape, generator=g).to(torch.bfloat16).cuda()
    # the last calls alone
    o_ref, l_ref = h.attn_fwd(q2, x["k"], x["v"], causal=causal)
    g_ref = h.attn_bwd(q2, x["k"], x["v"], o_ref, l_ref, do2, causal=causal)
    torch.cuda.synchronize()
    # the same calls behind others that write the same buffers
    out = torch.empty_like(o_ref)
    lse = torch.empty_like(l_ref)
    ws = torch.empty(h.bwd_workspace_size(w.B, w.Hq, w.Sq), dtype=torch.uint8, device="cuda")
    dq, dk, dv = (torch.empty_like(t) for t in g_ref)
    for rep in range(3):
        qq, dd = (x["q"], x["dout"]) if rep < 2 else (q2, do2)
        h.attn_fwd(qq, x["k"], x["v"], causal=causal, out=out, lse=lse)
        h.attn_bwd(qq, x["k"], x["v"], out, lse, dd, causal=causal, workspace=ws, dq=dq, dk=dk, dv=dv)
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    assert torch.equal(out.view(torch.int16), o_ref.view(torch.int16)) and torch.equal(lse, l_ref)
    for a, b in zip((dq, dk, dv), g_ref):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_dq_overlapping_the_dkdv_tail_repeats_bitwise(h):
    # 512 dK/dV units of 32 steps on 148 SMs (3.46 waves): the dQ kernel's CTAs
    # start on SMs the dK/dV tail leaves idle and take their units from the
    # counter, so which CTA computes which dQ tile varies from run to run; the
    # sums do not.  Three runs agree bitwise; one sampled row block of one head
    # against the oracle, dK / dV by the sums over keys.
    w = Workload("tail", B=1, Hq=16, Hkv=16, Sq=4096, Sk=4096, causal=False, seed=92)
    x_cpu = make_bwd_inputs(w)
    x = {k: v.cuda() for k, v in x_cpu.items()}
    out, lse = h.attn_fwd(x["q"], x["k"], x["v"])
    runs = [h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"]) for _ in range(3)]
    assert h.get_device_error() == 0
    for other in runs[1:]:
        for a, b in zip(runs[0], other):
            assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    dq, dk, dv = runs[0]
    dk_err = dk.double().sum(dim=2).abs() / dk.double().abs().sum(dim=2)
    dv_err = (dv.double().sum(dim=2) - x["dout"].double().sum(dim=2)).abs() / dv.double().abs().sum(dim=2)
    assert dk_err.max().item() <= 1e-2 and dv_err.max().item() <= 1e-2
    # dQ rows 0..127 of head 5 from the oracle on that head alone (dQ of a row
    # needs only its own query, dO and the head's K and V)
    hd, rows = 5, slice(0, 128)
    one = {n: x_cpu[n][:, hd:hd + 1] for n in ("q", "k", "v", "dout")}
    one["q"] = one["q"][:, :, rows]
    one["dout"] = one["dout"][:, :, rows]
    rdq, _, _, _, _ = oracle.attn_bwd(*(np_bits(one[n]) for n in ("q", "k", "v", "dout")), w.scale)
    e = grad_errors(dq[:, hd:hd + 1, rows], rdq)
    assert grad_ok(e), e
