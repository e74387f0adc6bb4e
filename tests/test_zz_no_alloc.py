"""attn_bwd_noalloc: the backward for callers that cannot allocate device
memory when they call us (a plug-in inside a framework that owns the GPU
allocator, or an engine whose memory is planned up front).  Its Delta scratch
is a static device array inside the library instead of a caller workspace.

The GPU test calls it through the C ABI twice in a row, on two different
problems, and checks each result against the workspace-taking attn_bwd with
the gradient tolerance the parity tests use (max abs <= 2e-2 * max(1, max|ref|),
normalised RMS <= 1e-2); both run the same kernels, so the results are also
expected to be bit-identical.  A second GPU case fills the static array to
its last row (B*Hq*Sq equal to the limit) and compares bit for bit with
attn_bwd.  This file is collected last on purpose.
"""
import ctypes

import pytest
import torch

from parity import grad_errors, grad_ok
from workloads import Workload, make_bwd_inputs


def _h():
    from head_attention_qk_b200 import build

    build.build()
    import head_attention_qk_b200 as h

    return h


def test_noalloc_refuses_problems_beyond_the_static_scratch():
    h = _h()
    A = ctypes.c_void_p(0x10000)
    rows = h.NOALLOC_MAX_ROWS
    # B*Hq*Sq = max + 128 rows: refused on the host, nothing launched
    rc = h.lib.attn_bwd_noalloc(A, A, A, A, A, A, A, A, A, 1, 1, 1, rows + 128, rows + 128, 128, 0.088, 0, None)
    assert rc == -4
    rc = h.lib.attn_bwd_noalloc(A, A, A, A, A, A, None, A, A, 1, 1, 1, 128, 128, 128, 0.088, 0, None)
    assert rc == -1


@pytest.mark.gpu
def test_noalloc_matches_workspace_backward_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    h = _h()
    problems = [Workload("na1", B=2, Hq=4, Hkv=2, Sq=300, Sk=300, causal=True, seed=401),
                Workload("na2", B=1, Hq=8, Hkv=2, Sq=200, Sk=333, causal=False, seed=402)]
    for w in problems:
        x = {k: v.cuda() for k, v in make_bwd_inputs(w).items()}
        out, lse = h.attn_fwd(x["q"], x["k"], x["v"], causal=w.causal)
        rdq, rdk, rdv = h.attn_bwd(x["q"], x["k"], x["v"], out, lse, x["dout"], causal=w.causal)
        dq, dk, dv = torch.empty_like(x["q"]), torch.empty_like(x["k"]), torch.empty_like(x["v"])
        p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
        rc = h.lib.attn_bwd_noalloc(p(x["q"]), p(x["k"]), p(x["v"]), p(out), p(lse), p(x["dout"]), p(dq), p(dk),
                                    p(dv), w.B, w.Hq, w.Hkv, w.Sq, w.Sk, w.D, w.scale, int(w.causal),
                                    ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
        assert rc == 0, h.lib.attn_error_string(rc)
        torch.cuda.synchronize()
        assert h.get_device_error() == 0
        for name, g, r in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
            e = grad_errors(g, r.double().cpu().numpy())
            assert grad_ok(e), (w.name, name, e)
            assert torch.equal(g.view(torch.int16), r.view(torch.int16)), (w.name, name)


@pytest.mark.gpu
def test_noalloc_at_the_row_limit_matches_workspace_backward():
    # B*Hq*Sq == HATTN_NOALLOC_MAX_ROWS: 2048 query heads of 2048 rows against
    # 128 keys each, so Delta fills the whole static array up to its last row
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    h = _h()
    B, H, Sq, Sk = 1, 2048, 2048, 128
    assert B * H * Sq == h.NOALLOC_MAX_ROWS
    g = torch.Generator(device="cuda").manual_seed(403)
    q, dout = (torch.randn(B, H, Sq, 128, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2))
    k, v = (torch.randn(B, H, Sk, 128, generator=g, device="cuda").to(torch.bfloat16) for _ in range(2))
    out, lse = h.attn_fwd(q, k, v)
    rdq, rdk, rdv = h.attn_bwd(q, k, v, out, lse, dout)
    dq, dk, dv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    p = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    rc = h.lib.attn_bwd_noalloc(p(q), p(k), p(v), p(out), p(lse), p(dout), p(dq), p(dk), p(dv), B, H, H, Sq, Sk,
                                128, 1.0 / 128 ** 0.5, 0, ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert rc == 0, h.lib.attn_error_string(rc)
    torch.cuda.synchronize()
    assert h.get_device_error() == 0
    for name, a, b in (("dq", dq, rdq), ("dk", dk, rdk), ("dv", dv, rdv)):
        assert torch.equal(a.view(torch.int16), b.view(torch.int16)), name
