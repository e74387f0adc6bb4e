"""Seeded input generators (CPU, torch.Generator).

Recipe (the same for the GPU path and the oracle):
- values are fp32 draws from N(0, 1) of a CPU ``torch.Generator`` seeded per
  workload, rounded to bf16 (round-to-nearest-even, torch's cast);
- Q, K, V (and dO for the backward) are drawn in that order from one generator;
  with ``per_row_seed`` each batch row b has its own generator seeded
  ``seed + b``, so a B=4 batch holds the B=2 batch in rows 0-1 bit for bit;
- ``qk_rmsnorm``: Q and K are normalised per token and per head over D,
  x / sqrt(mean(x^2) + 1e-6), no weight, in fp32, before the bf16 cast;
- e4m3: the bf16 values are quantised per (batch, head): descale = amax / 448,
  code = e4m3fn(clamp(x / descale, -448, 448)) with torch's round-to-nearest-even
  cast; the fp32 descales travel with the codes.
"""
from __future__ import annotations

import numpy as np
import torch

from .configs import Workload

E4M3_MAX = 448.0


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def _randn(shape, g: torch.Generator) -> torch.Tensor:
    return torch.randn(*shape, generator=g, dtype=torch.float32)


def rms_normalize(x: torch.Tensor, eps: float = 1e-6) -> torch.Tensor:
    """Per-token, per-head RMS normalisation over the last (head) dimension, fp32, no weight."""
    x = x.float()
    return x * torch.rsqrt(x.pow(2).mean(dim=-1, keepdim=True) + eps)


def quantize_e4m3_per_head(x: torch.Tensor):
    """[B,H,S,D] -> (e4m3fn codes [B,H,S,D], fp32 descale [B,H]) with descale = amax/448."""
    xf = x.float()
    amax = xf.abs().amax(dim=(2, 3))
    descale = torch.where(amax > 0, amax / E4M3_MAX, torch.ones_like(amax)).float()
    scaled = (xf / descale[:, :, None, None]).clamp(-E4M3_MAX, E4M3_MAX)
    return scaled.to(torch.float8_e4m3fn), descale


def _draw(w: Workload, B: int, shapes, n_tensors: int):
    """Draw n_tensors fp32 tensors of per-row shapes shapes[i] (each [H,S,D])."""
    if w.per_row_seed:
        rows = []
        for b in range(B):
            g = _gen(w.seed + b)
            rows.append([_randn(shapes[i], g) for i in range(n_tensors)])
        return [torch.stack([rows[b][i] for b in range(B)]) for i in range(n_tensors)]
    g = _gen(w.seed)
    return [_randn((B,) + tuple(shapes[i]), g) for i in range(n_tensors)]


def make_fwd_inputs(w: Workload, B: int | None = None):
    """Forward inputs on the CPU: dict(q, k, v[, q_descale, k_descale, v_descale]).

    bf16 workloads give bf16 tensors; e4m3 workloads give float8_e4m3fn tensors
    plus fp32 descales of shapes [B,Hq], [B,Hkv], [B,Hkv].
    """
    B = w.B if B is None else B
    shapes = [(w.Hq, w.Sq, w.D), (w.Hkv, w.Sk, w.D), (w.Hkv, w.Sk, w.D)]
    q, k, v = _draw(w, B, shapes, 3)
    if w.qk_rmsnorm:
        q, k = rms_normalize(q), rms_normalize(k)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    out = {"q": q, "k": k, "v": v}
    if w.dtype == "e4m3":
        for name in ("q", "k", "v"):
            codes, ds = quantize_e4m3_per_head(out[name])
            out[name] = codes
            out[name + "_descale"] = ds
    return out


def make_bwd_inputs(w: Workload, B: int | None = None):
    """Backward inputs (bf16): dict(q, k, v, dout)."""
    B = w.B if B is None else B
    shapes = [(w.Hq, w.Sq, w.D), (w.Hkv, w.Sk, w.D), (w.Hkv, w.Sk, w.D), (w.Hq, w.Sq, w.D)]
    q, k, v, do = _draw(w, B, shapes, 4)
    if w.qk_rmsnorm:
        q, k = rms_normalize(q), rms_normalize(k)
    return {n: t.to(torch.bfloat16) for n, t in zip(("q", "k", "v", "dout"), (q, k, v, do))}


def make_kvblock_inputs(w: Workload, n_blocks: int | None = None, block_len: int | None = None,
                        text_len: int | None = None):
    """Streaming inputs (bf16): q [B,Hq,Sq,D], blocks = list of (k_b, v_b) [B,Hkv,len,D],
    and the text cross-attention keys/values [B,Hkv,text_len,D]."""
    n_blocks = w.n_blocks if n_blocks is None else n_blocks
    block_len = (w.Sk // max(w.n_blocks, 1)) if block_len is None else block_len
    text_len = w.text_len if text_len is None else text_len
    g = _gen(w.seed)
    q = _randn((w.B, w.Hq, w.Sq, w.D), g).to(torch.bfloat16)
    blocks = []
    for _ in range(n_blocks):
        kb = _randn((w.B, w.Hkv, block_len, w.D), g).to(torch.bfloat16)
        vb = _randn((w.B, w.Hkv, block_len, w.D), g).to(torch.bfloat16)
        blocks.append((kb, vb))
    text = None
    if text_len:
        tk = _randn((w.B, w.Hkv, text_len, w.D), g).to(torch.bfloat16)
        tv = _randn((w.B, w.Hkv, text_len, w.D), g).to(torch.bfloat16)
        text = (tk, tv)
    return {"q": q, "blocks": blocks, "text": text}


def sample_rows(Sq: int, n: int = 256, seed: int = 0) -> np.ndarray:
    """A seeded sample of min(n, Sq) distinct query rows, sorted ascending."""
    perm = torch.randperm(Sq, generator=_gen(seed))[: min(n, Sq)]
    return np.sort(perm.numpy().astype(np.int64))


def bf16_bits(t: torch.Tensor) -> np.ndarray:
    """bf16 tensor -> numpy uint16 array of its bit patterns (no copy of values' meaning)."""
    assert t.dtype == torch.bfloat16
    return t.contiguous().view(torch.int16).numpy().view(np.uint16)


def e4m3_bits(t: torch.Tensor) -> np.ndarray:
    """float8_e4m3fn tensor -> numpy uint8 array of its codes."""
    assert t.dtype == torch.float8_e4m3fn
    return t.contiguous().view(torch.uint8).numpy()
