"""GPU parity of the forward (bf16 and e4m3) against the CPU fp64 oracle, plus
the bitwise properties: repeat runs, batch composition, head slicing, and
canary bytes around the outputs.

Bars: bf16 max |dO| <= 2e-2, max |dLSE| <= 1e-3 and normalised RMS of O
<= 1e-2 (at long Sk the outputs are small, |O| ~ 1e-2, so the max-abs bar
alone would let a badly wrong P V pass; bf16 rounding of O alone is ~0.3 %);
e4m3 normalised RMS of O <= 1e-2 against the oracle on the dequantized
inputs.  The long configs are checked on 256 seeded query rows per head.
"""
import math

import numpy as np
import pytest
import torch

import workloads
from parity import FP8_NRMS, LSE_MAX_ABS, O_MAX_ABS, O_NRMS, fwd_errors, oracle_fwd
from workloads import Workload, make_fwd_inputs, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def cuda(d):
    return {k: (v.cuda() if isinstance(v, torch.Tensor) else v) for k, v in d.items()}


def run_fwd(h, x, causal):
    ds = {}
    if x["q"].dtype == torch.float8_e4m3fn:
        ds = dict(q_descale=x["q_descale"], k_descale=x["k_descale"], v_descale=x["v_descale"])
    out, lse = h.attn_fwd(x["q"], x["k"], x["v"], causal=causal, **ds)
    assert h.get_device_error() == 0
    return out, lse


def check_bf16(h, w, rows=None):
    x_cpu = make_fwd_inputs(w)
    x = cuda(x_cpu)
    out, lse = run_fwd(h, x, w.causal)
    o_ref, lse_ref = oracle_fwd(x_cpu["q"], x_cpu["k"], x_cpu["v"], w.scale, w.causal, rows=rows)
    e = fwd_errors(out, lse, o_ref, lse_ref, rows)
    assert e["o_max_abs"] <= O_MAX_ABS and e["lse_max_abs"] <= LSE_MAX_ABS and e["o_nrms"] <= O_NRMS, e
    return e


# ------------------------------------------------------------------ small / ragged, full compare

def test_tiny_config(h):
    check_bf16(h, workloads.get("tiny"))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (1, 1, 1, 1, 1, False),
    (1, 2, 1, 1, 300, False),
    (2, 4, 2, 77, 300, False),
    (1, 2, 2, 300, 77, False),          # Sq > Sk without a mask
    (2, 4, 1, 257, 513, False),
    (1, 4, 2, 1000, 1000, True),
    (2, 2, 2, 129, 1100, True),         # causal, Sq < Sk (bottom-right)
    (1, 2, 2, 640, 640, True),
    (1, 40, 40, 600, 512, False),       # cross-attention shape, even head count
])
def test_ragged_shapes(h, B, Hq, Hkv, Sq, Sk, causal):
    w = Workload("ragged", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, seed=100 + Sq + Sk)
    check_bf16(h, w)


# More units (256 query rows x one (b, h)) than SMs and at most 8 KV tiles, no
# mask: these launch the persistent kernel (one CTA per SM looping over units).
@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk", [
    (1, 40, 40, 1560, 512),
    (2, 32, 8, 1000, 300),
    (2, 48, 16, 520, 1024),
])
def test_persistent_short_kv(h, B, Hq, Hkv, Sq, Sk):
    check_bf16(h, Workload("persist", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, seed=500 + Sq + Sk))


def test_persistent_causal_ragged(h):
    # causal with at most 16 KV tiles and more units than SMs: persistent, units
    # of unequal length dealt in snake order; ragged tails, Sq < Sk, 5 query heads per KV head
    check_bf16(h, Workload("persist_causal", B=2, Hq=40, Hkv=8, Sq=1000, Sk=1100, causal=True, seed=611))


def test_persistent_causal_matches_one_cta_per_unit_bitwise(h):
    # 320 units run persistently; one batch row of two heads (8 units) runs one CTA per unit
    w = Workload("persist_causal_bits", B=2, Hq=40, Hkv=8, Sq=1000, Sk=1100, causal=True, seed=612)
    x = cuda(make_fwd_inputs(w))
    o, l = run_fwd(h, x, True)
    xs = {"q": x["q"][1:, 5:7].contiguous(), "k": x["k"][1:, 1:2].contiguous(), "v": x["v"][1:, 1:2].contiguous()}
    o2, l2 = run_fwd(h, xs, True)
    assert torch.equal(o2.view(torch.int16), o[1:, 5:7].view(torch.int16))
    assert torch.equal(l2, l[1:, 5:7])


def test_persistent_matches_one_cta_per_unit_bitwise(h):
    # 280 units run persistently; three heads alone (21 units) run one CTA per unit
    w = Workload("persist_bits", B=1, Hq=40, Hkv=40, Sq=1560, Sk=512, seed=77)
    x = cuda(make_fwd_inputs(w))
    o, l = run_fwd(h, x, False)
    xs = {n: x[n][:, :3].contiguous() for n in ("q", "k", "v")}
    o3, l3 = run_fwd(h, xs, False)
    assert torch.equal(o3.view(torch.int16), o[:, :3].view(torch.int16))
    assert torch.equal(l3, l[:, :3])


def test_llm_config_sampled_rows(h):
    w = workloads.get("llm_gqa")
    check_bf16(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


def test_video_config_sampled_rows(h):
    w = workloads.get("video")
    check_bf16(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


def test_cross_attention_long_q_sampled_rows(h):
    # Sq >> Sk with an even head count (AITER PR #2911, Wan 2.2 cross-attention report)
    w = workloads.get("cross")
    check_bf16(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


def test_window_sink_shape_sampled_rows(h):
    # the raw SDPA call on the window-30 shape, 4680 queries against 51480 keys,
    # 12 heads (FlashDreams issue #739, SDPA kernels on gfx950)
    w = workloads.get("window")
    check_bf16(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


# ------------------------------------------------------------------ e4m3

def check_fp8(h, w, rows=None):
    x_cpu = make_fwd_inputs(w)
    x = cuda(x_cpu)
    out, lse = run_fwd(h, x, w.causal)
    o_ref, lse_ref = oracle_fwd(x_cpu["q"], x_cpu["k"], x_cpu["v"], w.scale, w.causal, rows=rows,
                                descales=(x_cpu["q_descale"], x_cpu["k_descale"], x_cpu["v_descale"]))
    e = fwd_errors(out, lse, o_ref, lse_ref, rows)
    assert e["o_nrms"] <= FP8_NRMS, e
    assert np.isfinite(e["lse_max_abs"]) and e["lse_max_abs"] < 5e-2, e
    return e


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (1, 2, 2, 256, 256, False),
    (2, 4, 2, 333, 517, False),
    (1, 2, 1, 700, 700, True),
    (1, 4, 2, 130, 700, True),          # causal, Sq < Sk, grouped heads
    (1, 2, 2, 1, 1, False),             # a single key
    (2, 2, 1, 5, 300, False),
])
def test_fp8_small(h, B, Hq, Hkv, Sq, Sk, causal):
    check_fp8(h, Workload("f8", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, dtype="e4m3", seed=Sq))


def test_fp8_persistent_short_kv(h):
    check_fp8(h, Workload("f8p", B=1, Hq=40, Hkv=20, Sq=1200, Sk=640, dtype="e4m3", seed=41))


def test_fp8_persistent_causal_ragged(h):
    # the persistent causal path (more units than SMs, at most 16 KV tiles) with e4m3 inputs
    check_fp8(h, Workload("f8pc", B=2, Hq=40, Hkv=8, Sq=1000, Sk=1100, causal=True, dtype="e4m3", seed=42))


def test_fp8_at_video_shape_sampled_rows(h):
    # the e4m3 bench line at the 32760-token video shape (Q, K RMS-normalised)
    w = workloads.get("fp8_32760")
    check_fp8(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


def test_bf16_at_fp8_shape_sampled_rows(h):
    # the bf16 bench line at the 75600-token shape
    w = workloads.get("bf16_75600")
    check_bf16(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


@pytest.mark.parametrize("B,Hq,Hkv,Sq,Sk,causal", [
    (1, 4, 2, 333, 517, False),
    (1, 4, 2, 700, 900, True),
    (1, 40, 20, 1200, 640, False),      # persistent, short KV
    (2, 40, 8, 1000, 1100, True),       # persistent causal
    (1, 2, 2, 1, 1, False),
])
def test_fp8_entry_points_agree_bitwise(h, B, Hq, Hkv, Sq, Sk, causal):
    # attn_fwd widens each e4m3 V tile in shared memory inside the attention
    # kernel (nothing allocated), attn_fwd_ws (the binding's path) widens V
    # into the caller's scratch first: the same fp16 values reach the same
    # MMAs, so the results are the same bits
    import ctypes

    w = Workload("f8ws", B=B, Hq=Hq, Hkv=Hkv, Sq=Sq, Sk=Sk, causal=causal, dtype="e4m3", seed=23 + Sq)
    x = cuda(make_fwd_inputs(w))
    o1, l1 = run_fwd(h, x, causal)
    o2 = torch.empty_like(o1)
    l2 = torch.empty_like(l1)
    P = lambda t: ctypes.c_void_p(t.data_ptr())
    rc = h.lib.attn_fwd(P(x["q"]), P(x["k"]), P(x["v"]), P(o2), P(l2), B, Hq, Hkv, Sq, Sk, 128, w.scale,
                        int(causal), 1, P(x["q_descale"]), P(x["k_descale"]), P(x["v_descale"]),
                        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_fp8_config_sampled_rows(h):
    w = workloads.get("fp8")
    check_fp8(h, w, rows=sample_rows(w.Sq, 256, seed=w.seed))


# ------------------------------------------------------------------ bitwise properties

def test_repeat_runs_are_bitwise_equal(h):
    w = workloads.get("llm_gqa")
    x = cuda(make_fwd_inputs(w))
    o1, l1 = run_fwd(h, x, True)
    o2, l2 = run_fwd(h, x, True)
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l1.view(torch.int32), l2.view(torch.int32))


def test_batch_composition_is_bitwise_invariant(h):
    w = workloads.get("llm_gqa")
    x2 = cuda(make_fwd_inputs(w, B=2))
    x4 = cuda(make_fwd_inputs(w, B=4))
    assert torch.equal(x4["q"][:2], x2["q"])                  # same rows by construction
    o2, l2 = run_fwd(h, x2, True)
    o4, l4 = run_fwd(h, x4, True)
    assert torch.equal(o4[:2].view(torch.int16), o2.view(torch.int16))
    assert torch.equal(l4[:2], l2)
    x1 = {k: v[1:2].contiguous() for k, v in x2.items()}      # one row at a time
    o1, l1 = run_fwd(h, x1, True)
    assert torch.equal(o1.view(torch.int16), o2[1:2].view(torch.int16))


def test_head_slice_is_bitwise_invariant(h):
    # a tensor-parallel rank holding query heads 8..15 and their KV heads 2..3
    w = workloads.get("llm_gqa", B=1)
    x = cuda(make_fwd_inputs(w, B=1))
    o, l = run_fwd(h, x, True)
    xs = {"q": x["q"][:, 8:16].contiguous(), "k": x["k"][:, 2:4].contiguous(), "v": x["v"][:, 2:4].contiguous()}
    os_, ls = run_fwd(h, xs, True)
    assert torch.equal(os_.view(torch.int16), o[:, 8:16].view(torch.int16))
    assert torch.equal(ls, l[:, 8:16])


def test_outputs_leave_neighbouring_bytes_untouched(h):
    w = Workload("canary", B=1, Hq=2, Hkv=2, Sq=200, Sk=333, seed=9)
    x = cuda(make_fwd_inputs(w))
    pad = 4096
    o_buf = torch.full((pad + 2 * 200 * 128 + pad,), -12345, dtype=torch.int16, device="cuda")
    l_buf = torch.full((pad + 2 * 200 + pad,), float("nan"), dtype=torch.float32, device="cuda")
    out = o_buf[pad:pad + 2 * 200 * 128].view(torch.bfloat16).view(1, 2, 200, 128)
    lse = l_buf[pad:pad + 400].view(1, 2, 200)
    h.attn_fwd(x["q"], x["k"], x["v"], out=out, lse=lse)
    assert h.get_device_error() == 0
    assert torch.all(o_buf[:pad] == -12345) and torch.all(o_buf[-pad:] == -12345)
    assert torch.all(torch.isnan(l_buf[:pad])) and torch.all(torch.isnan(l_buf[-pad:]))
    assert torch.all(torch.isfinite(lse))


def test_closed_forms_on_gpu(h):
    # identical keys: O = mean(V), LSE = ln Sk + scale q.k; zero queries: LSE = ln Sk
    Sk = 777
    g = torch.Generator().manual_seed(11)
    q = torch.randn(1, 2, 130, 128, generator=g).to(torch.bfloat16)
    k1 = torch.randn(1, 2, 1, 128, generator=g).to(torch.bfloat16)
    k = k1.expand(1, 2, Sk, 128).contiguous()
    v = torch.randn(1, 2, Sk, 128, generator=g).to(torch.bfloat16)
    out, lse = h.attn_fwd(q.cuda(), k.cuda(), v.cuda())
    scale = 1 / math.sqrt(128)
    mean_v = v.double().mean(dim=2, keepdim=True)
    assert (out.double().cpu() - mean_v).abs().max() <= O_MAX_ABS
    assert ((out.double().cpu() - mean_v).norm() / mean_v.expand_as(out).norm()) <= O_NRMS
    expect = math.log(Sk) + scale * torch.einsum("bhid,bhd->bhi", q.double(), k1[:, :, 0].double())
    assert (lse.double().cpu() - expect).abs().max() <= LSE_MAX_ABS
    out0, lse0 = h.attn_fwd(torch.zeros_like(q).cuda(), k.cuda(), v.cuda())
    assert (lse0.double().cpu() - math.log(Sk)).abs().max() <= LSE_MAX_ABS
