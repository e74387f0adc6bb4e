"""Helpers shared by the GPU parity tests: run the oracle on the same bytes the
GPU read, and measure the distance between the two.

Tolerances (restated in the tests that use them):
- bf16 forward: max |O_gpu - O_ref| <= 2e-2 and max |LSE_gpu - LSE_ref| <= 1e-3;
- e4m3 forward: ||O_gpu - O_ref||_2 / ||O_ref||_2 <= 1e-2 against the oracle on
  the dequantized inputs;
- backward (no tolerance given on the pages): for each of dQ, dK, dV,
  max abs <= 2e-2 * max(1, max |ref|) and normalised RMS <= 1e-2;
- e4m3 prologue (the pages fix no precision for the norm; the kernel computes
  it in fp32, the oracle in fp64): descales within a relative 2^-17 of the
  oracle's; codes equal except where the oracle's fp64 quotient y / descale
  lies within a relative 2^-16 of an e4m3 rounding midpoint, and there they
  differ by exactly one code step with the same sign.  Both bounds come from
  the fp32 error of the kernel's steps: a sum of 128 non-negative squares in
  any order is within 127 u of the exact sum (u = 2^-24), so the row factor
  1 / sqrt(ss / 128 + eps) is within about 67 u, y within 68 u, the descale
  within 70 u (< 2^-17) and the fp32 quotient within 139 u (< 2^-16).
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
O_NRMS = 1e-2
E4M3_DESCALE_REL = 2.0 ** -17
E4M3_BOUNDARY_REL = 2.0 ** -16


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


def e4m3_midpoints() -> np.ndarray:
    """The rounding boundaries of e4m3fn: midpoints between neighbouring
    non-negative finite values (codes 0x00..0x7E, decoded by torch's float8 type)."""
    vals = torch.arange(0x7F, dtype=torch.uint8).view(torch.float8_e4m3fn).double().numpy()
    return (vals[:-1] + vals[1:]) / 2


def near_e4m3_boundary(q: np.ndarray, rel: float) -> np.ndarray:
    """True where |q| lies within relative distance rel of an e4m3 rounding midpoint."""
    mids = e4m3_midpoints()
    a = np.abs(np.asarray(q, dtype=np.float64))
    idx = np.searchsorted(mids, a)
    lo = mids[np.clip(idx - 1, 0, mids.size - 1)]
    hi = mids[np.clip(idx, 0, mids.size - 1)]
    d = np.minimum(np.abs(a - lo) / lo, np.abs(a - hi) / hi)
    return d <= rel


def check_e4m3_codes(got_codes, got_descale, ref_codes, ref_descale, ref_quotient,
                     descale_rel=E4M3_DESCALE_REL, boundary_rel=E4M3_BOUNDARY_REL):
    """Apply the e4m3 parity rule; returns the number of codes that differ
    (each next to a rounding boundary and one step away).  Raises AssertionError."""
    got_descale = np.asarray(got_descale, dtype=np.float64)
    ref_descale = np.asarray(ref_descale, dtype=np.float64)
    rel = np.abs(got_descale / ref_descale - 1.0)
    assert np.all(rel <= descale_rel), ("descale", float(rel.max()))
    got = np.asarray(got_codes, dtype=np.uint8).ravel()
    ref = np.asarray(ref_codes, dtype=np.uint8).ravel()
    bad = np.flatnonzero(got != ref)
    if bad.size == 0:
        return 0
    g, r = got[bad].astype(np.int32), ref[bad].astype(np.int32)
    same_sign = (g & 0x80) == (r & 0x80)
    one_step = np.abs((g & 0x7F) - (r & 0x7F)) == 1
    near = near_e4m3_boundary(np.asarray(ref_quotient).ravel()[bad], boundary_rel)
    ok = same_sign & one_step & near
    assert np.all(ok), ("codes differ away from a rounding boundary", int((~ok).sum()), bad[~ok][:5],
                        g[~ok][:5], r[~ok][:5])
    return int(bad.size)
