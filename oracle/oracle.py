"""CPU fp64 attention oracle (ctypes wrapper around attn_oracle.c).

TEST INFRASTRUCTURE ONLY.  The test suite, the smoke check and the CPU-baseline
leg of the benchmark are the only callers.  The product library never imports
this module, and this module never imports the product library: the two share
no code.  Inputs are numpy arrays holding the same bytes the GPU reads:

* ``float64`` arrays (kind F64),
* ``uint16`` arrays of bfloat16 bit patterns (kind BF16),
* ``uint8`` arrays of OCP e4m3fn codes (kind E4M3) plus per-(batch, head)
  descales.

All arithmetic happens in double precision in C (see attn_oracle.c for the
definitions and the page sections they restate).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "attn_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

F64, BF16, E4M3 = 0, 1, 2


def compile_library(src: str, out: str) -> str:
    """Compile a C source of the oracle into a shared library at `out` (gcc,
    OpenMP, no fast-math, no contraction of multiply-adds)."""
    tmp = out + ".tmp.%d" % os.getpid()
    cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-std=c11",
           "-Wall", "-shared", "-fPIC", "-o", tmp, src, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, out)
    return out


def source_path() -> str:
    """Path of the oracle's C source."""
    return _SRC


def build(force: bool = False) -> str:
    """Compile attn_oracle.c into liboracle.so next to it (gcc, OpenMP, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    return compile_library(_SRC, _LIB)


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(os.environ.get("ORACLE_LIB") or build())
            vp, dp, i64p = ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p
            ci, cd = ctypes.c_int, ctypes.c_double
            lib.oracle_attn_fwd.argtypes = [ci, vp, vp, vp, dp, dp, dp, ci, ci, ci, ci, ci, ci,
                                            cd, ci, i64p, ci, dp, dp]
            lib.oracle_attn_fwd.restype = ci
            lib.oracle_lse_merge.argtypes = [dp, dp, ci, ctypes.c_int64, ci, dp, dp]
            lib.oracle_lse_merge.restype = ci
            lib.oracle_attn_bwd.argtypes = [ci, vp, vp, vp, vp, ci, ci, ci, ci, ci, ci, cd, ci,
                                            dp, dp, dp, dp, dp]
            lib.oracle_attn_bwd.restype = ci
            lib.oracle_e4m3_to_double.argtypes = [ctypes.c_uint8]
            lib.oracle_e4m3_to_double.restype = cd
            lib.oracle_num_threads.argtypes = []
            lib.oracle_num_threads.restype = ci
            lib.oracle_e4m3_rne.argtypes = [ctypes.c_double]
            lib.oracle_e4m3_rne.restype = ctypes.c_uint8
            lib.oracle_quantize_e4m3.argtypes = [vp, vp, vp, vp, ci, ci, ci, ci, ci, cd]
            lib.oracle_quantize_e4m3.restype = ci
            _lib = lib
    return _lib


def _kind(a: np.ndarray) -> int:
    if a.dtype == np.float64:
        return F64
    if a.dtype == np.uint16:
        return BF16
    if a.dtype == np.uint8:
        return E4M3
    raise TypeError("oracle inputs must be float64, uint16 (bf16 bits) or uint8 (e4m3 codes), got %s" % a.dtype)


def _ptr(a):
    return None if a is None else a.ctypes.data


def num_threads() -> int:
    return _load().oracle_num_threads()


def e4m3_to_double(code: int) -> float:
    return _load().oracle_e4m3_to_double(int(code) & 0xFF)


def e4m3_rne(v: float) -> int:
    """e4m3fn code of a real value: nearest, ties to the even code, saturating at +-448."""
    return int(_load().oracle_e4m3_rne(float(v)))


def quantize_e4m3(x_bits, rmsnorm=False, eps=1e-6, with_quotient=False):
    """e4m3 prologue (see attn_oracle.c): bf16 bits [B,H,S,D] -> (codes uint8 [B,H,S,D],
    descale float32 [B,H]); with_quotient also returns the fp64 quotients
    y / descale [B,H,S,D] that the codes round."""
    x_bits = np.ascontiguousarray(x_bits)
    if x_bits.dtype != np.uint16 or x_bits.ndim != 4:
        raise TypeError("quantize_e4m3 takes [B,H,S,D] uint16 bf16 bit patterns")
    B, H, S, D = x_bits.shape
    codes = np.empty(x_bits.shape, dtype=np.uint8)
    descale = np.empty((B, H), dtype=np.float32)
    quot = np.empty(x_bits.shape, dtype=np.float64) if with_quotient else None
    rc = _load().oracle_quantize_e4m3(_ptr(x_bits), _ptr(codes), _ptr(descale), _ptr(quot), B, H, S, D,
                                      int(bool(rmsnorm)), float(eps))
    if rc != 0:
        raise RuntimeError("oracle_quantize_e4m3 failed with code %d" % rc)
    return (codes, descale, quot) if with_quotient else (codes, descale)


def attn_fwd(q, k, v, scale, causal=False, rows=None, descales=None):
    """O and LSE for the query rows ``rows`` (all rows if None).

    q: [B,Hq,Sq,D]; k, v: [B,Hkv,Sk,D]; same storage kind for all three.
    descales: (q_descale [B,Hq], k_descale [B,Hkv], v_descale [B,Hkv]) for e4m3.
    Returns o [B,Hq,n_rows,D] float64 and lse [B,Hq,n_rows] float64.
    """
    q, k, v = (np.ascontiguousarray(x) for x in (q, k, v))
    kind = _kind(q)
    if _kind(k) != kind or _kind(v) != kind:
        raise TypeError("q, k, v must share one storage kind")
    B, Hq, Sq, D = q.shape
    Bk, Hkv, Sk, Dk = k.shape
    if v.shape != k.shape or Bk != B or Dk != D:
        raise ValueError("shape mismatch")
    if rows is None:
        rows_arr = None
        n_rows = Sq
    else:
        rows_arr = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        n_rows = int(rows_arr.size)
        if n_rows and (rows_arr.min() < 0 or rows_arr.max() >= Sq):
            raise ValueError("row index out of range")
    dq_ = dk_ = dv_ = None
    if kind == E4M3:
        if descales is None:
            raise ValueError("e4m3 inputs need descales")
        dq_, dk_, dv_ = (np.ascontiguousarray(np.asarray(x, dtype=np.float64)) for x in descales)
        if dq_.size != B * Hq or dk_.size != B * Hkv or dv_.size != B * Hkv:
            raise ValueError("descale shape mismatch")
    o = np.empty((B, Hq, n_rows, D), dtype=np.float64)
    lse = np.empty((B, Hq, n_rows), dtype=np.float64)
    rc = _load().oracle_attn_fwd(kind, _ptr(q), _ptr(k), _ptr(v), _ptr(dq_), _ptr(dk_), _ptr(dv_),
                                 B, Hq, Hkv, Sq, Sk, D, float(scale), int(bool(causal)),
                                 _ptr(rows_arr), n_rows, _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError("oracle_attn_fwd failed with code %d" % rc)
    return o, lse


def lse_merge(o_parts, lse_parts):
    """Fold per-block (O_b, LSE_b) in ascending block order.

    o_parts: [n_blocks, ..., D]; lse_parts: [n_blocks, ...] (same leading dims).
    Returns o [..., D], lse [...].
    """
    o_parts = np.ascontiguousarray(o_parts, dtype=np.float64)
    lse_parts = np.ascontiguousarray(lse_parts, dtype=np.float64)
    n = o_parts.shape[0]
    D = o_parts.shape[-1]
    rows = int(np.prod(o_parts.shape[1:-1]))
    if lse_parts.shape != o_parts.shape[:-1]:
        raise ValueError("shape mismatch")
    o = np.empty(o_parts.shape[1:], dtype=np.float64)
    lse = np.empty(lse_parts.shape[1:], dtype=np.float64)
    rc = _load().oracle_lse_merge(_ptr(o_parts), _ptr(lse_parts), n, rows, D, _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError("oracle_lse_merge failed with code %d" % rc)
    return o, lse


def attn_bwd(q, k, v, dout, scale, causal=False):
    """dQ, dK, dV (and the oracle's own O, LSE) in float64."""
    q, k, v, dout = (np.ascontiguousarray(x) for x in (q, k, v, dout))
    kind = _kind(q)
    if kind == E4M3 or any(_kind(x) != kind for x in (k, v, dout)):
        raise TypeError("backward takes float64 or bf16 inputs of one kind")
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    dq = np.empty(q.shape, dtype=np.float64)
    dk = np.empty(k.shape, dtype=np.float64)
    dv = np.empty(v.shape, dtype=np.float64)
    o = np.empty(q.shape, dtype=np.float64)
    lse = np.empty((B, Hq, Sq), dtype=np.float64)
    rc = _load().oracle_attn_bwd(kind, _ptr(q), _ptr(k), _ptr(v), _ptr(dout), B, Hq, Hkv, Sq, Sk, D,
                                 float(scale), int(bool(causal)), _ptr(dq), _ptr(dk), _ptr(dv),
                                 _ptr(o), _ptr(lse))
    if rc != 0:
        raise RuntimeError("oracle_attn_bwd failed with code %d" % rc)
    return dq, dk, dv, o, lse
