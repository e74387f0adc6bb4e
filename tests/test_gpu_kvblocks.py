"""GPU parity of the block-KV streaming forward (per-block partials merged by
LSE in ascending block order) against the oracle: the oracle computes each
block and merges with its own fp64 fold, and also runs the unsplit attention.

Bars as for the bf16 forward: max |dO| <= 2e-2, max |dLSE| <= 1e-3 and
normalised RMS of O <= 1e-2.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import LSE_MAX_ABS, O_MAX_ABS, O_NRMS, fwd_errors, np_bits, oracle_fwd
from workloads import Workload, make_kvblock_inputs, sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def bf16_ok(e):
    return e["o_max_abs"] <= O_MAX_ABS and e["lse_max_abs"] <= LSE_MAX_ABS and e["o_nrms"] <= O_NRMS


def check_blocks(h, q, blocks, rows=None):
    kb = [k.cuda() for k, _ in blocks]
    vb = [v.cuda() for _, v in blocks]
    out, lse = h.attn_fwd_kvblocks(q.cuda(), kb, vb)
    assert h.get_device_error() == 0
    scale = 1.0 / np.sqrt(q.shape[-1])
    parts = [oracle_fwd(q, k, v, scale, rows=rows) for k, v in blocks]
    o_m, lse_m = oracle.lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    e = fwd_errors(out, lse, o_m, lse_m, rows)
    assert bf16_ok(e), e
    k_all = torch.cat([k for k, _ in blocks], dim=2)
    v_all = torch.cat([v for _, v in blocks], dim=2)
    o_u, lse_u = oracle_fwd(q, k_all, v_all, scale, rows=rows)
    e2 = fwd_errors(out, lse, o_u, lse_u, rows)
    assert bf16_ok(e2), e2
    return out, lse


@pytest.mark.parametrize("lens", [[128], [100, 300], [1, 129, 77, 256], [640] * 3])
def test_kvblocks_ragged(h, lens):
    w = Workload("kb", B=2, Hq=4, Hkv=2, Sq=200, Sk=sum(lens), seed=300 + len(lens))
    g = torch.Generator().manual_seed(w.seed)
    q = torch.randn(2, 4, 200, 128, generator=g).to(torch.bfloat16)
    blocks = [(torch.randn(2, 2, n, 128, generator=g).to(torch.bfloat16),
               torch.randn(2, 2, n, 128, generator=g).to(torch.bfloat16)) for n in lens]
    check_blocks(h, q, blocks)


def test_kvblocks_more_blocks_than_one_launch(h):
    g = torch.Generator().manual_seed(31)
    q = torch.randn(1, 2, 130, 128, generator=g).to(torch.bfloat16)
    blocks = [(torch.randn(1, 2, 40 + i, 128, generator=g).to(torch.bfloat16),
               torch.randn(1, 2, 40 + i, 128, generator=g).to(torch.bfloat16)) for i in range(37)]
    check_blocks(h, q, blocks)


def test_kvblocks_persistent_short_blocks(h):
    # 5 query pairs x 40 heads = 200 units (> 148 SMs), each folding 3 blocks
    # of 8 KV tiles in all: the persistent kernel
    g = torch.Generator().manual_seed(57)
    q = torch.randn(1, 40, 1200, 128, generator=g).to(torch.bfloat16)
    blocks = [(torch.randn(1, 8, n, 128, generator=g).to(torch.bfloat16),
               torch.randn(1, 8, n, 128, generator=g).to(torch.bfloat16)) for n in (512, 77, 300)]
    out, lse = check_blocks(h, q, blocks, rows=sample_rows(1200, 64, seed=57))
    # the same query heads in a launch too small to run persistently: bitwise equal
    o5, l5 = h.attn_fwd_kvblocks(q[:, :5].contiguous().cuda(), [k[:, :1].contiguous().cuda() for k, _ in blocks],
                                 [v[:, :1].contiguous().cuda() for _, v in blocks])
    assert torch.equal(o5.view(torch.int16), out[:, :5].view(torch.int16)) and torch.equal(l5, lse[:, :5])


def test_streaming_config(h):
    w = workloads.get("streaming")
    x = make_kvblock_inputs(w)
    rows = sample_rows(w.Sq, 256, seed=w.seed)
    out, lse = check_blocks(h, x["q"], x["blocks"], rows=rows)
    # repeat: bitwise
    out2, lse2 = h.attn_fwd_kvblocks(x["q"].cuda(), [k.cuda() for k, _ in x["blocks"]],
                                     [v.cuda() for _, v in x["blocks"]])
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)) and torch.equal(lse, lse2)
    # cross-attention of the same queries to the text tokens
    tk, tv = x["text"]
    o_t, l_t = h.attn_fwd(x["q"].cuda(), tk.cuda(), tv.cuda())
    o_ref, l_ref = oracle_fwd(x["q"], tk, tv, w.scale)
    e = fwd_errors(o_t, l_t, o_ref, l_ref)
    assert bf16_ok(e), e


@pytest.mark.parametrize("n_window", [20, 40])
def test_sink_and_window_frames_as_block_list(h, n_window):
    # A frame-major KV cache (each frame of 1560 latent tokens is its own
    # contiguous [B, Hkv, 1560, D] block) attended through a sink + window
    # selection: the first frame plus the last n_window frames, passed as a list
    # of non-contiguous cache blocks (FlashDreams issue #739, window-30 SDPA
    # with sink frames; FlashDreams PR #486 section 1.2, caller-managed block
    # KV cache).  21 blocks fold inside one launch, 41 take the partials and
    # merge path.  Compared with the oracle on the concatenated keys.
    w = workloads.get("window")
    frames, L = n_window + 12, 1560
    g = torch.Generator().manual_seed(w.seed + n_window)
    q = torch.randn(w.B, w.Hq, w.Sq, w.D, generator=g).to(torch.bfloat16)
    cache_k = torch.randn(frames, w.B, w.Hkv, L, w.D, generator=g).to(torch.bfloat16)
    cache_v = torch.randn(frames, w.B, w.Hkv, L, w.D, generator=g).to(torch.bfloat16)
    picked = [0] + list(range(frames - n_window, frames))
    ck, cv = cache_k.cuda(), cache_v.cuda()
    ws = torch.empty(h.kvblocks_workspace_size(w.B, w.Hq, w.Sq, w.D, len(picked)) or 1, dtype=torch.uint8,
                     device="cuda")
    out, lse = h.attn_fwd_kvblocks(q.cuda(), [ck[f] for f in picked], [cv[f] for f in picked], workspace=ws)
    assert h.get_device_error() == 0
    rows = sample_rows(w.Sq, 256, seed=w.seed)
    k_all = torch.cat([cache_k[f] for f in picked], dim=2)
    v_all = torch.cat([cache_v[f] for f in picked], dim=2)
    o_ref, lse_ref = oracle_fwd(q, k_all, v_all, w.scale, rows=rows)
    e = fwd_errors(out, lse, o_ref, lse_ref, rows)
    assert bf16_ok(e), e
