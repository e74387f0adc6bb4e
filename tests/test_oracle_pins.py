"""Pins for the CPU fp64 oracle, independent of the oracle itself.

Each check is fixed by the mathematics or by a library routine, not by the
oracle's own code: closed forms (single key, identical keys, zero queries),
split-and-merge equals unsplit, an independent brute-force loop with
math.fsum, torch's fp64 SDPA and autograd, central finite differences for the
backward, invariants, and the e4m3/bf16 decodings against torch's casts.
"""
import math

import numpy as np
import pytest
import torch

from workloads import bf16_bits, e4m3_bits, quantize_e4m3_per_head, sample_rows

pytestmark = pytest.mark.filterwarnings("ignore")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ---------------------------------------------------------------- closed forms

def test_single_key_gives_v0_and_score(oracle_mod):
    q, k, v = rnd((1, 3, 5, 16), 1), rnd((1, 3, 1, 16), 2), rnd((1, 3, 1, 16), 3)
    scale = 0.37
    o, lse = oracle_mod.attn_fwd(q, k, v, scale)
    for h in range(3):
        for i in range(5):
            np.testing.assert_allclose(o[0, h, i], v[0, h, 0], rtol=0, atol=1e-15)
            s0 = scale * math.fsum(q[0, h, i] * k[0, h, 0])
            assert abs(lse[0, h, i] - s0) < 1e-13


def test_identical_keys_mean_v_and_log_sk(oracle_mod):
    Sk, D = 37, 8
    q = rnd((2, 2, 4, D), 4)
    k = np.broadcast_to(rnd((2, 2, 1, D), 5), (2, 2, Sk, D)).copy()
    v = rnd((2, 2, Sk, D), 6)
    scale = 1 / math.sqrt(D)
    o, lse = oracle_mod.attn_fwd(q, k, v, scale)
    mean_v = v.mean(axis=2)
    for b in range(2):
        for h in range(2):
            for i in range(4):
                np.testing.assert_allclose(o[b, h, i], mean_v[b, h], atol=1e-14)
                expect = math.log(Sk) + scale * math.fsum(q[b, h, i] * k[b, h, 0])
                assert abs(lse[b, h, i] - expect) < 1e-13


def test_zero_q_gives_log_sk(oracle_mod):
    Sk = 300
    q = np.zeros((1, 2, 3, 8))
    k, v = rnd((1, 2, Sk, 8), 7), rnd((1, 2, Sk, 8), 8)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5)
    np.testing.assert_allclose(lse, math.log(Sk), atol=1e-13)
    np.testing.assert_allclose(o, np.broadcast_to(v.mean(axis=2)[:, :, None, :], o.shape), atol=1e-14)


def test_bwd_single_key(oracle_mod):
    q, k, v, do = rnd((1, 2, 6, 8), 9), rnd((1, 2, 1, 8), 10), rnd((1, 2, 1, 8), 11), rnd((1, 2, 6, 8), 12)
    dq, dk, dv, o, _ = oracle_mod.attn_bwd(q, k, v, do, 0.3)
    assert np.abs(dq).max() < 1e-14 and np.abs(dk).max() < 1e-14
    np.testing.assert_allclose(dv[:, :, 0], do.sum(axis=2), atol=1e-13)


def test_bwd_identical_keys(oracle_mod):
    Sk = 9
    q = rnd((1, 1, 5, 8), 13)
    k = np.broadcast_to(rnd((1, 1, 1, 8), 14), (1, 1, Sk, 8)).copy()
    v, do = rnd((1, 1, Sk, 8), 15), rnd((1, 1, 5, 8), 16)
    dq, dk, dv, _, _ = oracle_mod.attn_bwd(q, k, v, do, 0.4)
    assert np.abs(dq).max() < 1e-13
    for j in range(Sk):
        np.testing.assert_allclose(dv[0, 0, j], do[0, 0].sum(axis=0) / Sk, atol=1e-14)


# ---------------------------------------------------------------- split / merge

@pytest.mark.parametrize("cuts", [[5], [1, 7, 20], [13, 14, 30, 31]])
def test_split_merge_equals_unsplit(oracle_mod, cuts):
    Sk = 40
    q, k, v = rnd((2, 4, 6, 16), 17), rnd((2, 2, Sk, 16), 18), rnd((2, 2, Sk, 16), 19)
    scale = 0.25
    o_ref, lse_ref = oracle_mod.attn_fwd(q, k, v, scale)
    edges = [0] + cuts + [Sk]
    parts = [oracle_mod.attn_fwd(q, k[:, :, a:b], v[:, :, a:b], scale) for a, b in zip(edges[:-1], edges[1:])]
    o, lse = oracle_mod.lse_merge(np.stack([p[0] for p in parts]), np.stack([p[1] for p in parts]))
    np.testing.assert_allclose(o, o_ref, rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref, rtol=0, atol=1e-12)


def test_merge_skips_empty_block(oracle_mod):
    o_parts = rnd((3, 4, 8), 20)
    lse_parts = rnd((3, 4), 21)
    lse_parts[1, :] = -np.inf
    o, lse = oracle_mod.lse_merge(o_parts, lse_parts)
    o2, lse2 = oracle_mod.lse_merge(o_parts[[0, 2]], lse_parts[[0, 2]])
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


# ---------------------------------------------------------------- brute force

def brute_force(q, k, v, scale, causal):
    """Independent loop: weights normalised by an explicit fsum, LSE via log(fsum)."""
    B, Hq, Sq, D = q.shape
    Hkv, Sk = k.shape[1], k.shape[2]
    G = Hq // Hkv
    o = np.zeros((B, Hq, Sq, D))
    lse = np.zeros((B, Hq, Sq))
    for b in range(B):
        for h in range(Hq):
            kh = h // G
            for i in range(Sq):
                keys = [j for j in range(Sk) if (not causal) or j <= i + Sk - Sq]
                if not keys:
                    lse[b, h, i] = -math.inf
                    continue
                sc = [scale * math.fsum(q[b, h, i, d] * k[b, kh, j, d] for d in range(D)) for j in keys]
                mx = max(sc)
                e = [math.exp(s - mx) for s in sc]
                tot = math.fsum(e)
                lse[b, h, i] = mx + math.log(tot)
                for d in range(D):
                    o[b, h, i, d] = math.fsum(e[t] / tot * v[b, kh, j, d] for t, j in enumerate(keys))
    return o, lse


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(8, 8), (5, 7), (3, 8)])
def test_brute_force_tiny(oracle_mod, causal, Sq, Sk):
    q, k, v = rnd((2, 4, Sq, 4), 22), rnd((2, 2, Sk, 4), 23), rnd((2, 2, Sk, 4), 24)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.6, causal=causal)
    o2, lse2 = brute_force(q, k, v, 0.6, causal)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


def test_fully_masked_rows_are_zero(oracle_mod):
    # causal with Sq > Sk (bottom-right aligned): the first Sq - Sk rows see no key
    q, k, v = rnd((1, 1, 6, 4), 25), rnd((1, 1, 4, 4), 26), rnd((1, 1, 4, 4), 27)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, causal=True)
    assert np.all(o[0, 0, :2] == 0) and np.all(np.isneginf(lse[0, 0, :2]))
    assert np.all(np.isfinite(lse[0, 0, 2:]))
    o2, lse2 = brute_force(q, k, v, 0.5, True)
    np.testing.assert_allclose(o, o2, atol=1e-13)


# ---------------------------------------------------------------- library routines

def torch_ref(q, k, v, scale, causal):
    qt, kt, vt = (torch.from_numpy(x) for x in (q, k, v))
    G = qt.shape[1] // kt.shape[1]
    kt, vt = kt.repeat_interleave(G, dim=1), vt.repeat_interleave(G, dim=1)
    Sq, Sk = qt.shape[2], kt.shape[2]
    mask = None
    if causal:
        mask = torch.ones(Sq, Sk, dtype=torch.bool).tril(diagonal=Sk - Sq)
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale)
    s = torch.einsum("bhid,bhjd->bhij", qt, kt) * scale
    if mask is not None:
        s = s.masked_fill(~mask, -math.inf)
    return o.numpy(), torch.logsumexp(s, dim=-1).numpy()


@pytest.mark.parametrize("causal", [False, True])
@pytest.mark.parametrize("Sq,Sk", [(64, 64), (33, 90)])
def test_matches_torch_sdpa_fp64(oracle_mod, causal, Sq, Sk):
    q, k, v = rnd((2, 8, Sq, 32), 28), rnd((2, 2, Sk, 32), 29), rnd((2, 2, Sk, 32), 30)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.2, causal=causal)
    o2, lse2 = torch_ref(q, k, v, 0.2, causal)
    np.testing.assert_allclose(o, o2, atol=1e-12)
    np.testing.assert_allclose(lse, lse2, atol=1e-12)


@pytest.mark.parametrize("causal", [False, True])
def test_bwd_matches_torch_autograd_fp64(oracle_mod, causal):
    q, k, v, do = rnd((1, 4, 24, 16), 31), rnd((1, 2, 40, 16), 32), rnd((1, 2, 40, 16), 33), rnd((1, 4, 24, 16), 34)
    dq, dk, dv, o, lse = oracle_mod.attn_bwd(q, k, v, do, 0.3, causal=causal)
    qt, kt, vt = (torch.from_numpy(x).requires_grad_(True) for x in (q, k, v))
    G = 2
    mask = torch.ones(24, 40, dtype=torch.bool).tril(diagonal=16) if causal else None
    ot = torch.nn.functional.scaled_dot_product_attention(
        qt, kt.repeat_interleave(G, 1), vt.repeat_interleave(G, 1), attn_mask=mask, scale=0.3)
    ot.backward(torch.from_numpy(do))
    np.testing.assert_allclose(o, ot.detach().numpy(), atol=1e-12)
    np.testing.assert_allclose(dq, qt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dk, kt.grad.numpy(), atol=1e-11)
    np.testing.assert_allclose(dv, vt.grad.numpy(), atol=1e-11)


# ---------------------------------------------------------------- finite differences

@pytest.mark.parametrize("causal", [False, True])
def test_bwd_central_differences(oracle_mod, causal):
    B, Hq, Hkv, Sq, Sk, D = 1, 2, 1, 3, 4, 3
    q, k, v, do = rnd((B, Hq, Sq, D), 35), rnd((B, Hkv, Sk, D), 36), rnd((B, Hkv, Sk, D), 37), rnd((B, Hq, Sq, D), 38)
    scale, h = 0.7, 1e-6
    dq, dk, dv, _, _ = oracle_mod.attn_bwd(q, k, v, do, scale, causal=causal)

    def loss(q, k, v):
        o, _ = oracle_mod.attn_fwd(q, k, v, scale, causal=causal)
        return math.fsum((o * do).ravel())

    base = {"q": q, "k": k, "v": v}
    for name, grad in (("q", dq), ("k", dk), ("v", dv)):
        arr = base[name]
        for idx in np.ndindex(arr.shape):
            plus, minus = arr.copy(), arr.copy()
            plus[idx] += h
            minus[idx] -= h
            fd = (loss(**{**base, name: plus}) - loss(**{**base, name: minus})) / (2 * h)
            assert abs(fd - grad[idx]) <= 1e-6 * max(1.0, abs(grad[idx])), (name, idx, fd, grad[idx])


# ---------------------------------------------------------------- invariants

def test_rows_of_p_sum_to_one(oracle_mod):
    q, k = rnd((1, 2, 9, 8), 39), rnd((1, 2, 11, 8), 40)
    for causal in (False, True):
        o, _ = oracle_mod.attn_fwd(q, k, np.ones((1, 2, 11, 8)), 0.9, causal=causal)
        np.testing.assert_allclose(o, 1.0, atol=1e-14)


def test_causal_row0_sees_key0(oracle_mod):
    q, k, v = rnd((1, 2, 7, 8), 41), rnd((1, 2, 7, 8), 42), rnd((1, 2, 7, 8), 43)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, causal=True)
    np.testing.assert_allclose(o[:, :, 0], v[:, :, 0], atol=1e-15)


def test_key_value_permutation_invariance(oracle_mod):
    q, k, v = rnd((1, 2, 5, 8), 44), rnd((1, 2, 19, 8), 45), rnd((1, 2, 19, 8), 46)
    perm = np.random.default_rng(47).permutation(19)
    o, lse = oracle_mod.attn_fwd(q, k, v, 0.5)
    o2, lse2 = oracle_mod.attn_fwd(q, k[:, :, perm], v[:, :, perm], 0.5)
    np.testing.assert_allclose(o, o2, atol=1e-13)
    np.testing.assert_allclose(lse, lse2, atol=1e-13)


def test_gqa_equals_duplicated_mha(oracle_mod):
    q, k, v = rnd((2, 6, 5, 8), 48), rnd((2, 2, 9, 8), 49), rnd((2, 2, 9, 8), 50)
    for causal in (False, True):
        o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, causal=causal)
        o2, lse2 = oracle_mod.attn_fwd(q, np.repeat(k, 3, axis=1), np.repeat(v, 3, axis=1), 0.5, causal=causal)
        np.testing.assert_array_equal(o, o2)
        np.testing.assert_array_equal(lse, lse2)


def test_row_sampling_matches_full(oracle_mod):
    q, k, v = rnd((1, 3, 50, 8), 51), rnd((1, 3, 50, 8), 52), rnd((1, 3, 50, 8), 53)
    rows = sample_rows(50, 12, seed=5)
    for causal in (False, True):
        o, lse = oracle_mod.attn_fwd(q, k, v, 0.5, causal=causal)
        os_, lses = oracle_mod.attn_fwd(q, k, v, 0.5, causal=causal, rows=rows)
        np.testing.assert_array_equal(os_, o[:, :, rows])
        np.testing.assert_array_equal(lses, lse[:, :, rows])


# ---------------------------------------------------------------- storage decodings

def test_e4m3_decoding_matches_torch_cast(oracle_mod):
    codes = torch.arange(256, dtype=torch.int32).to(torch.uint8)
    ref = codes.view(torch.float8_e4m3fn).to(torch.float64).numpy()
    for c in range(256):
        got = oracle_mod.e4m3_to_double(c)
        if np.isnan(ref[c]):
            assert math.isnan(got), c
        else:
            assert got == ref[c], (c, got, ref[c])
    assert oracle_mod.e4m3_to_double(0x7E) == 448.0


def test_bf16_storage_is_exact_widening(oracle_mod):
    g = torch.Generator().manual_seed(54)
    q, k, v = (torch.randn(1, 2, 33, 16, generator=g).to(torch.bfloat16) for _ in range(3))
    o, lse = oracle_mod.attn_fwd(bf16_bits(q), bf16_bits(k), bf16_bits(v), 0.25, causal=True)
    o2, lse2 = oracle_mod.attn_fwd(*(t.double().numpy() for t in (q, k, v)), 0.25, causal=True)
    np.testing.assert_array_equal(o, o2)
    np.testing.assert_array_equal(lse, lse2)


@pytest.mark.parametrize("Hq,Hkv", [(3, 3), (6, 2)])
def test_e4m3_storage_applies_per_head_descale(oracle_mod, Hq, Hkv):
    # heads of different magnitudes, so every (batch, head) has its own descale;
    # with grouped heads the query descales are per query head, not per KV head
    g = torch.Generator().manual_seed(55 + Hq)
    mag = lambda H: torch.arange(1, 2 * H + 1, dtype=torch.float32).reshape(2, H, 1, 1)
    x = [(torch.randn(2, H, 21, 16, generator=g) * mag(H)).to(torch.bfloat16) for H in (Hq, Hkv, Hkv)]
    (q8, dq), (k8, dk), (v8, dv) = (quantize_e4m3_per_head(t) for t in x)
    assert len(set(dq.flatten().tolist())) == 2 * Hq
    o, lse = oracle_mod.attn_fwd(e4m3_bits(q8), e4m3_bits(k8), e4m3_bits(v8), 0.25,
                                 descales=(dq.numpy(), dk.numpy(), dv.numpy()))
    deq = [c.to(torch.float64) * d.double()[:, :, None, None] for c, d in ((q8, dq), (k8, dk), (v8, dv))]
    o2, lse2 = oracle_mod.attn_fwd(*(t.numpy() for t in deq), 0.25)
    np.testing.assert_allclose(o, o2, rtol=0, atol=1e-15)
    np.testing.assert_allclose(lse, lse2, rtol=0, atol=1e-15)
