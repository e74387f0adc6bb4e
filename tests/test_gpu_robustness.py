"""Failure detection, CUDA-graph capture and fail-closed behaviour on the GPU.

- A kernel whose wait can never be satisfied gives up after a short limit,
  reports the site in the device error word, and the context stays usable.
- The forward and backward calls allocate nothing and never synchronise, so
  they can be captured into a CUDA graph; replay equals the eager results bit
  for bit.  The e4m3 forward without a workspace leaves device memory as it was.
- Unsupported requests raise instead of being approximated.
- Calls on a stream that is not torch's current one keep their outputs and
  scratch to that stream: allocations on the current stream meanwhile cannot
  take them over while the kernels still use them.
"""
import ctypes

import pytest
import torch

import workloads
from parity import LSE_MAX_ABS, O_MAX_ABS, fwd_errors, oracle_fwd
from workloads import Workload, make_bwd_inputs, make_fwd_inputs, make_kvblock_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def test_bounded_wait_gives_up_and_context_survives(h):
    assert h.get_device_error() == 0
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert h.lib.attn_selftest_bounded_wait(stream, 100_000) == 0        # 100 ms limit
    assert h.get_device_error() == 0x17F                                  # 0x100 | self-test site
    assert h.get_device_error() == 0                                      # read clears the word
    # the context is still usable: a normal forward is correct afterwards
    w = Workload("after", B=1, Hq=2, Hkv=2, Sq=200, Sk=300, seed=77)
    x = make_fwd_inputs(w)
    out, lse = h.attn_fwd(x["q"].cuda(), x["k"].cuda(), x["v"].cuda())
    assert h.get_device_error() == 0
    o_ref, lse_ref = oracle_fwd(x["q"], x["k"], x["v"], w.scale)
    e = fwd_errors(out, lse, o_ref, lse_ref)
    assert e["o_max_abs"] <= O_MAX_ABS and e["lse_max_abs"] <= LSE_MAX_ABS


def test_counter_wait_gives_up_and_context_survives(h):
    # the bounded wait the one-pass backward orders its dQ additions with: a
    # counter that nothing increments, a 100 ms limit
    counter = torch.zeros(1, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert h.get_device_error() == 0
    assert h.lib.attn_selftest_counter_wait(ctypes.c_void_p(counter.data_ptr()), stream, 100_000) == 0
    assert h.get_device_error() == 0x12A                                  # 0x100 | ordered-add site
    assert h.get_device_error() == 0
    w = Workload("after2", B=1, Hq=2, Hkv=1, Sq=300, Sk=300, causal=True, seed=76)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out, lse = h.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    dq, dk, dv = h.attn_bwd_onepass(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    dq2, dk2, dv2 = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True)
    assert h.get_device_error() == 0
    assert (dq.float() - dq2.float()).abs().max() < 2e-2


def test_selftest_rejects_bad_limits(h):
    assert h.lib.attn_selftest_bounded_wait(None, 0) == -1
    assert h.lib.attn_selftest_bounded_wait(None, 20_000_000) == -1
    assert h.lib.attn_selftest_counter_wait(None, None, 1000) == -1


def test_cuda_graph_capture_matches_eager(h):
    w = Workload("graph", B=2, Hq=4, Hkv=2, Sq=333, Sk=333, causal=True, seed=78)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out_e, lse_e = h.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    dq_e, dk_e, dv_e = h.attn_bwd(x["q"], x["k"], x["v"], out_e, lse_e, x["dout"], causal=True)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            out_g, lse_g = h.attn_fwd(x["q"], x["k"], x["v"], causal=True, stream=s)
            dq_g, dk_g, dv_g = h.attn_bwd(x["q"], x["k"], x["v"], out_g, lse_g, x["dout"], causal=True, stream=s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    for a, b in ((out_g, out_e), (dq_g, dq_e), (dk_g, dk_e), (dv_g, dv_e)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(lse_g, lse_e)


def test_cuda_graph_llm_step_replays_bitwise(h):
    # the LLM step (B2 Hq32 Hkv8 S2048 causal, forward + backward) in one graph:
    # the backward's dQ grid starts while dK/dV still runs and takes its units
    # from a counter in the workspace that the Delta kernel resets, so replays
    # queued back to back, with no sync between them, must each start from a
    # reset counter; every replay equals the eager step bit for bit
    import workloads

    w = workloads.get("llm_gqa")
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    out_e, lse_e = h.attn_fwd(x["q"], x["k"], x["v"], causal=True)
    grads_e = h.attn_bwd(x["q"], x["k"], x["v"], out_e, lse_e, x["dout"], causal=True)
    torch.cuda.synchronize()
    ws = torch.empty(h.bwd_workspace_size(w.B, w.Hq, w.Sq), dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            out_g, lse_g = h.attn_fwd(x["q"], x["k"], x["v"], causal=True, stream=s)
            grads_g = h.attn_bwd(x["q"], x["k"], x["v"], out_g, lse_g, x["dout"], causal=True, workspace=ws,
                                 stream=s)
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16)) and torch.equal(lse_g, lse_e)
    for a, b in zip(grads_g, grads_e):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16))


def test_fp8_attn_fwd_allocates_nothing_and_captures(h):
    # the C attn_fwd with e4m3 inputs and no workspace widens V inside the
    # kernel: no device memory changes hands (an fp16 copy of this V would be
    # 64 MB), and the call captures into a graph whose replays equal the eager
    # result
    w = Workload("graph8", B=1, Hq=4, Hkv=2, Sq=300, Sk=131072, dtype="e4m3", seed=79)
    x = {k: v.cuda() for k, v in make_fwd_inputs(w).items()}
    P = lambda t: ctypes.c_void_p(t.data_ptr())

    def call(out, lse, stream):
        return h.lib.attn_fwd(P(x["q"]), P(x["k"]), P(x["v"]), P(out), P(lse), 1, 4, 2, 300, w.Sk, 128, w.scale, 0,
                              1, P(x["q_descale"]), P(x["k_descale"]), P(x["v_descale"]),
                              ctypes.c_void_p(stream.cuda_stream))

    out_e = torch.empty(1, 4, 300, 128, dtype=torch.bfloat16, device="cuda")
    lse_e = torch.empty(1, 4, 300, dtype=torch.float32, device="cuda")
    assert call(out_e, lse_e, torch.cuda.current_stream()) == 0      # first call: module load, kernel setup
    torch.cuda.synchronize()
    free0 = torch.cuda.mem_get_info()[0]
    for _ in range(3):
        assert call(out_e, lse_e, torch.cuda.current_stream()) == 0
        assert torch.cuda.mem_get_info()[0] == free0                   # nothing taken while enqueued
    torch.cuda.synchronize()
    assert torch.cuda.mem_get_info()[0] == free0
    assert h.get_device_error() == 0
    out_g = torch.zeros_like(out_e)
    lse_g = torch.zeros_like(lse_e)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            assert call(out_g, lse_g, s) == 0
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16)) and torch.equal(lse_g, lse_e)
    del g


def test_cuda_graph_capture_prologue_then_fp8(h):
    # the e4m3 prologue (memset + two kernels) and the e4m3 forward on its
    # codes, captured in one graph; replays equal the eager calls bit for bit
    g0 = torch.Generator().manual_seed(80)
    q, k, v = (torch.randn(1, 3, S, 128, generator=g0).to(torch.bfloat16).cuda() for S in (250, 270, 270))
    ws = torch.empty(h.fwd_workspace_size(1, 3, 270, 128, h.E4M3), dtype=torch.uint8, device="cuda")

    def run(stream):
        qc, qd = h.quantize_e4m3(q, rmsnorm=True, stream=stream)
        kc, kd = h.quantize_e4m3(k, rmsnorm=True, stream=stream)
        vc, vd = h.quantize_e4m3(v, rmsnorm=False, stream=stream)
        out, lse = h.attn_fwd(qc, kc, vc, q_descale=qd, k_descale=kd, v_descale=vd, workspace=ws, stream=stream)
        return qc, qd, out, lse

    eager = run(None)
    torch.cuda.synchronize()
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(s):
        with torch.cuda.graph(g, stream=s):
            graphed = run(s)
    for _ in range(2):
        g.replay()
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    for a, b in zip(graphed, eager):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del g


def test_fail_closed_on_device(h):
    q = torch.zeros(1, 2, 64, 64, dtype=torch.bfloat16, device="cuda")     # head dim 64 is not offered
    with pytest.raises(h.HattnError) as ei:
        h.attn_fwd(q, q, q)
    assert ei.value.code == -2
    q = torch.zeros(1, 2, 64, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 2, 32, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(h.HattnError) as ei:
        h.attn_fwd(q, k, k, causal=True)                                    # causal with Sq > Sk
    assert ei.value.code == -2
    q8 = torch.zeros(1, 2, 64, 128, dtype=torch.float8_e4m3fn, device="cuda")
    with pytest.raises(h.HattnError) as ei:
        h.attn_fwd(q8, q8, q8)                                              # e4m3 without descales
    assert ei.value.code == -1
    assert h.get_device_error() == 0


def test_side_stream_eager_calls_keep_their_scratch(h):
    # Each call runs on a side stream s behind a ~50 ms spin, so its kernels
    # start long after it returns.  Right after each call the current stream
    # allocates buffers of the scratch's size and fills them: had the binding
    # taken the scratch on the current stream (and released it on return),
    # the fill would land in it before the kernels read it.  Results must
    # equal default-stream calls bit for bit.
    w = Workload("side", B=2, Hq=4, Hkv=2, Sq=700, Sk=900, causal=True, seed=81)
    x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
    w8 = Workload("side8", B=1, Hq=4, Hkv=2, Sq=500, Sk=600, dtype="e4m3", seed=82)
    x8 = {k: v.cuda() for k, v in make_fwd_inputs(w8).items()}
    ds8 = dict(q_descale=x8["q_descale"], k_descale=x8["k_descale"], v_descale=x8["v_descale"])
    kv = make_kvblock_inputs(Workload("side_kv", B=1, Hq=2, Hkv=2, Sq=130, Sk=37 * 40, seed=83),
                             n_blocks=37, block_len=40, text_len=0)
    qb, kb, vb = kv["q"].cuda(), [t.cuda() for t, _ in kv["blocks"]], [t.cuda() for _, t in kv["blocks"]]

    def run(stream):
        out, lse = h.attn_fwd(x["q"], x["k"], x["v"], causal=True, stream=stream)
        grads = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=True, stream=stream)
        o8, l8 = h.attn_fwd(x8["q"], x8["k"], x8["v"], stream=stream, **ds8)
        ob, lb = h.attn_fwd_kvblocks(qb, kb, vb, stream=stream)
        return (out, lse, o8, l8, ob, lb) + tuple(grads)

    ref = run(None)
    torch.cuda.synchronize()
    sizes = [h.bwd_workspace_size(2, 4, 700), h.fwd_workspace_size(1, 2, 600, 128, h.E4M3),
             h.kvblocks_workspace_size(1, 2, 130, 128, 37)]
    assert all(n > 0 for n in sizes)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        torch.cuda._sleep(100_000_000)
    got = run(s)
    junk = [torch.full((n,), 0x7F, dtype=torch.uint8, device="cuda") for n in sizes for _ in range(4)]
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    for a, b in zip(got, ref):
        assert torch.equal(a.view(torch.uint8), b.view(torch.uint8))
    del junk
