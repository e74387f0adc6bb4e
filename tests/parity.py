"""Helpers shared by the GPU parity tests: run the oracle on the same bytes the
GPU read, and measure the distance between the two.

Tolerances (restated in the tests that use them):
- bf16 forward: max |O_gpu - O_ref| <= 2e-2 and max |LSE_gpu - LSE_ref| <= 1e-3;
- e4m3 forward: ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 1e-2 against the oracle on
  the dequantized inputs;
- backward (no tolerance given on the pages): for each of dQ, dK, dV,
  max abs <= 2e-2 * max(1, max |ref|) and normalised RMS <= 1e-2.
"""
from __future__ import annotations

import numpy as np
import torch

import oracle
from workloads import bf16_bits, e4m3_bits

O_MAX_ABS = 2e-2
LSE_MAX_ABS = 1e-3
FP8_NRMS = 1e-2
GRAD_REL_MAX = 2e-2
GRAD_NRMS = 1e-2


def np_bits(t: torch.Tensor) -> np.ndarray:
    t = t.detach().cpu().contiguous()
    if t.dtype == torch.bfloat16:
        return bf16_bits(t)
    if t.dtype == torch.float8_e4m3fn:
        return e4m3_bits(t)
    raise TypeError(t.dtype)


def oracle_fwd(q, k, v, scale, causal=False, rows=None, descales=None):
    ds = None
    if descales is not None:
        ds = tuple(d.detach().cpu().double().numpy().ravel() for d in descales)
    return oracle.attn_fwd(np_bits(q), np_bits(k), np_bits(v), scale, causal=causal, rows=rows, descales=ds)


def nrms(a: np.ndarray, ref: np.ndarray) -> float:
    den = np.sqrt(np.sum(ref * ref))
    return float(np.sqrt(np.sum((a - ref) ** 2)) / den) if den > 0 else float(np.sqrt(np.sum(a * a)))


def fwd_errors(o_gpu: torch.Tensor, lse_gpu: torch.Tensor, o_ref, lse_ref, rows=None):
    o = o_gpu.detach().float().cpu().numpy().astype(np.float64)
    lse = lse_gpu.detach().cpu().numpy().astype(np.float64)
    if rows is not None:
        o, lse = o[:, :, rows], lse[:, :, rows]
    return {
        "o_max_abs": float(np.max(np.abs(o - o_ref))),
        "o_nrms": nrms(o, o_ref),
        "lse_max_abs": float(np.max(np.abs(lse - lse_ref))),
    }


def grad_errors(g_gpu: torch.Tensor, g_ref: np.ndarray):
    g = g_gpu.detach().float().cpu().numpy().astype(np.float64)
    return {"max_abs": float(np.max(np.abs(g - g_ref))), "ref_max": float(np.max(np.abs(g_ref))),
            "nrms": nrms(g, g_ref)}


def grad_ok(e) -> bool:
    return e["max_abs"] <= GRAD_REL_MAX * max(1.0, e["ref_max"]) and e["nrms"] <= GRAD_NRMS
