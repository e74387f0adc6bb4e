"""GPU parity of the block-KV forward over an FP8 (e4m3) KV cache whose blocks
carry their own per-head descales (FlashDreams PR #486 "flashdreams.accelerated
API v0", section 1.2: FP8 KV cache, streaming self-attention over a block KV
cache).  The cache is written the way a caller would write it: each new block
of bf16 keys / values quantised in place by the product prologue
(attn_quantize_e4m3 writing the block's codes and its B*Hkv descales into the
cache's slots).

The oracle runs on the same codes and descales, two ways: block by block with
its own fp64 merge, and on the concatenated keys dequantized by torch's float8
decoding (an fp64 attention over real values).  Bar: normalised RMS of O
<= 1e-2 (the FP8 bar); repeat runs are bitwise equal.
"""
import numpy as np
import pytest
import torch

import oracle
import workloads
from parity import FP8_NRMS, fwd_errors, np_bits, oracle_fwd
from workloads import sample_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h():
    if not torch.cuda.is_available():
        pytest.skip("needs a GPU")
    import head_attention_qk_b200 as pkg

    return pkg


def fp8_cache(h, q_bf16, blocks_bf16, rmsnorm_qk=False):
    """Quantise q and every (k, v) block with the product prologue into a
    frame-major e4m3 cache; returns device codes and descales."""
    B, Hq, Sq, D = q_bf16.shape
    n = len(blocks_bf16)
    Hkv = blocks_bf16[0][0].shape[1]
    qc, qd = h.quantize_e4m3(q_bf16.cuda(), rmsnorm=rmsnorm_qk)
    kds = torch.empty(n, B, Hkv, dtype=torch.float32, device="cuda")
    vds = torch.empty_like(kds)
    kc, vc = [], []
    for i, (kb, vb) in enumerate(blocks_bf16):
        ck = torch.empty(kb.shape, dtype=torch.float8_e4m3fn, device="cuda")
        cv = torch.empty(vb.shape, dtype=torch.float8_e4m3fn, device="cuda")
        h.quantize_e4m3(kb.cuda(), rmsnorm=rmsnorm_qk, codes=ck, descale=kds[i])
        h.quantize_e4m3(vb.cuda(), rmsnorm=False, codes=cv, descale=vds[i])
        kc.append(ck)
        vc.append(cv)
    return qc, qd, kc, vc, kds, vds


def dequant(codes, ds):
    """Real values of e4m3 codes [B,H,S,D] with per-(b,h) descales, in fp64 (torch decode)."""
    return codes.cpu().double() * ds.cpu().double().reshape(codes.shape[0], codes.shape[1], 1, 1)


def check_fp8_blocks(h, qc, qd, kc, vc, kds, vds, rows=None):
    out, lse = h.attn_fwd_kvblocks(qc, kc, vc, q_descale=qd, k_descale=kds, v_descale=vds)
    assert h.get_device_error() == 0
    scale = 1.0 / np.sqrt(qc.shape[-1])
    # block by block on the codes, merged by the oracle's fixed-order fold
    parts = [oracle_fwd(qc.cpu(), kc[i].cpu(), vc[i].cpu(), scale, rows=rows, descales=(qd, kds[i], vds[i]))
             for i in range(len(kc))]
    o_m, lse_m = oracle.lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    e = fwd_errors(out, lse, o_m, lse_m, rows)
    assert e["o_nrms"] <= FP8_NRMS, e
    # the whole key sequence, dequantized by torch, as fp64 values
    qr = dequant(qc, qd).numpy()
    kr = torch.cat([dequant(kc[i], kds[i]) for i in range(len(kc))], dim=2).numpy()
    vr = torch.cat([dequant(vc[i], vds[i]) for i in range(len(vc))], dim=2).numpy()
    o_u, lse_u = oracle.attn_fwd(qr, kr, vr, scale, rows=rows)
    e2 = fwd_errors(out, lse, o_u, lse_u, rows)
    assert e2["o_nrms"] <= FP8_NRMS and e2["lse_max_abs"] < 5e-2, e2
    return out, lse, e2


def _blocks(g, B, Hkv, lens, D=128, v_scales=None):
    out = []
    for i, n in enumerate(lens):
        sv = 1.0 if v_scales is None else v_scales[i]
        out.append((torch.randn(B, Hkv, n, D, generator=g).to(torch.bfloat16),
                    (torch.randn(B, Hkv, n, D, generator=g) * sv).to(torch.bfloat16)))
    return out


@pytest.mark.parametrize("lens", [[128], [100, 300], [1, 129, 77, 256], [640] * 3])
def test_fp8_kvblocks_ragged(h, lens):
    g = torch.Generator().manual_seed(700 + len(lens))
    q = torch.randn(2, 4, 200, 128, generator=g).to(torch.bfloat16)
    check_fp8_blocks(h, *fp8_cache(h, q, _blocks(g, 2, 2, lens)))


def test_fp8_kvblocks_unequal_v_scales(h):
    # V blocks of very different magnitudes: each block's probabilities enter
    # P V scaled by vd_b / max vd, the output by max vd
    g = torch.Generator().manual_seed(711)
    q = torch.randn(1, 4, 300, 128, generator=g).to(torch.bfloat16)
    blocks = _blocks(g, 1, 2, [200, 130, 333, 64], v_scales=[1.0, 1e-3, 40.0, 0.05])
    check_fp8_blocks(h, *fp8_cache(h, q, blocks))


def test_fp8_kvblocks_more_blocks_than_one_launch(h):
    g = torch.Generator().manual_seed(712)
    q = torch.randn(1, 2, 130, 128, generator=g).to(torch.bfloat16)
    check_fp8_blocks(h, *fp8_cache(h, q, _blocks(g, 1, 2, [40 + i for i in range(37)])))


def test_fp8_kvblocks_persistent_short_blocks(h):
    # 5 query pairs x 40 heads = 200 units (> 148 SMs), each folding 3 blocks
    # of 8 KV tiles in all: the persistent kernel
    g = torch.Generator().manual_seed(713)
    q = torch.randn(1, 40, 1200, 128, generator=g).to(torch.bfloat16)
    cache = fp8_cache(h, q, _blocks(g, 1, 8, [512, 77, 300]))
    out, lse, _ = check_fp8_blocks(h, *cache, rows=sample_rows(1200, 64, seed=713))
    qc, qd, kc, vc, kds, vds = cache
    # five query heads (one KV head) alone: too small to run persistently, bitwise equal
    o5, l5 = h.attn_fwd_kvblocks(qc[:, :5].contiguous(), [k[:, :1].contiguous() for k in kc],
                                 [v[:, :1].contiguous() for v in vc], q_descale=qd[:, :5].contiguous(),
                                 k_descale=kds[:, :, :1].contiguous(), v_descale=vds[:, :, :1].contiguous())
    assert torch.equal(o5.view(torch.int16), out[:, :5].view(torch.int16)) and torch.equal(l5, lse[:, :5])


def test_fp8_single_block_matches_attn_fwd_bitwise(h):
    # one block is the plain e4m3 forward
    g = torch.Generator().manual_seed(714)
    q = torch.randn(1, 4, 300, 128, generator=g).to(torch.bfloat16)
    qc, qd, kc, vc, kds, vds = fp8_cache(h, q, _blocks(g, 1, 2, [700]))
    o1, l1 = h.attn_fwd_kvblocks(qc, kc, vc, q_descale=qd, k_descale=kds, v_descale=vds)
    o2, l2 = h.attn_fwd(qc, kc[0], vc[0], q_descale=qd, k_descale=kds[0], v_descale=vds[0])
    assert torch.equal(o1.view(torch.int16), o2.view(torch.int16)) and torch.equal(l1, l2)


def test_fp8_streaming_config(h):
    # the streaming config with an FP8 cache: 1560 new-frame queries (Q, K
    # RMS-normalised in the prologue) against 21 cached blocks of 1560 keys,
    # each block quantised with its own descales; 256 rows per head
    w = workloads.get("streaming")
    x = workloads.make_kvblock_inputs(w)
    cache = fp8_cache(h, x["q"], x["blocks"], rmsnorm_qk=True)
    rows = sample_rows(w.Sq, 256, seed=w.seed)
    out, lse, e = check_fp8_blocks(h, *cache, rows=rows)
    qc, qd, kc, vc, kds, vds = cache
    out2, lse2 = h.attn_fwd_kvblocks(qc, kc, vc, q_descale=qd, k_descale=kds, v_descale=vds)
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16)) and torch.equal(lse, lse2)
