"""ctypes binding of libhattn.so (see include/hattn.h).

Argument marshalling only: every step of the attention computation runs in
the library's CUDA kernels.  PyTorch supplies device memory and the current
stream.  Importing this module raises if the compiled library is missing;
there is no fallback implementation.
"""
from __future__ import annotations

import ctypes
import math
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libhattn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError("libhattn.so is not built; run `python -m head_attention_qk_b200.build` "
                      "(nvcc for sm_100a) -- there is no non-CUDA fallback")

lib = ctypes.CDLL(LIB_PATH)

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.attn_fwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _vp, _vp, _vp]
lib.attn_fwd.restype = _i
lib.attn_fwd_ws.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _i, _vp, _vp, _vp, _vp, _sz, _vp]
lib.attn_fwd_ws.restype = _i
lib.attn_fwd_workspace_size.argtypes = [_i, _i, _i, _i, _i]
lib.attn_fwd_workspace_size.restype = _sz
lib.attn_fwd_kvblocks.argtypes = [_vp, _vp, _vp, _vp, _i, _vp, _vp, _i, _i, _i, _i, _i, _f, _i, _vp, _vp, _vp,
                                  _vp, _sz, _vp]
lib.attn_fwd_kvblocks.restype = _i
lib.attn_fwd_kvblocks_workspace_size.argtypes = [_i, _i, _i, _i, _i]
lib.attn_fwd_kvblocks_workspace_size.restype = _sz
lib.attn_bwd.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz, _vp]
lib.attn_bwd.restype = _i
lib.attn_bwd_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp]
lib.attn_bwd_noalloc.restype = _i
lib.attn_bwd_workspace_size.argtypes = [_i, _i, _i]
lib.attn_bwd_workspace_size.restype = _sz
lib.attn_get_device_error.argtypes = [_vp, ctypes.POINTER(_i)]
lib.attn_get_device_error.restype = _i
lib.attn_quantize_e4m3.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, _i, ctypes.c_double, _vp]
lib.attn_quantize_e4m3.restype = _i
lib.attn_selftest_bounded_wait.argtypes = [_vp, ctypes.c_uint]
lib.attn_selftest_bounded_wait.restype = _i
lib.attn_error_string.argtypes = [_i]
lib.attn_error_string.restype = ctypes.c_char_p

BF16, E4M3 = 0, 1
EXPORTED = ("attn_fwd", "attn_fwd_ws", "attn_fwd_workspace_size", "attn_quantize_e4m3", "attn_fwd_kvblocks", "attn_fwd_kvblocks_workspace_size", "attn_bwd",
            "attn_bwd_workspace_size", "attn_bwd_noalloc", "attn_get_device_error", "attn_selftest_bounded_wait",
            "attn_error_string")
NOALLOC_MAX_ROWS = 1 << 22


class HattnError(RuntimeError):
    def __init__(self, code: int, where: str):
        self.code = code
        super().__init__("%s failed: %d (%s)" % (where, code, lib.attn_error_string(code).decode()))


def _check(rc: int, where: str):
    if rc != 0:
        raise HattnError(rc, where)


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float8_e4m3fn:
        return E4M3
    raise TypeError("inputs must be bfloat16 or float8_e4m3fn, got %s" % t.dtype)


def _require(t: torch.Tensor, name: str):
    if not t.is_cuda:
        raise ValueError("%s must be a CUDA tensor" % name)
    if not t.is_contiguous():
        raise ValueError("%s must be contiguous" % name)


def fwd_workspace_size(B, Hkv, Sk, D, dtype) -> int:
    return lib.attn_fwd_workspace_size(B, Hkv, Sk, D, dtype)


def attn_fwd(q, k, v, causal=False, scale=None, q_descale=None, k_descale=None, v_descale=None,
             out=None, lse=None, workspace=None, stream=None):
    """O [B,Hq,Sq,D] bf16 and LSE [B,Hq,Sq] fp32 for q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D].

    e4m3 inputs need scratch for the fp16 copy of V: `workspace` (a CUDA byte
    tensor of at least fwd_workspace_size() bytes), else one from torch's
    allocator; the library itself then allocates nothing.
    """
    for t, n in ((q, "q"), (k, "k"), (v, "v")):
        _require(t, n)
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    dt = _dtype_code(q)
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    ws_bytes = fwd_workspace_size(B, Hkv, Sk, D, dt)
    if ws_bytes and workspace is None:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if workspace is not None:
        _require(workspace, "workspace")
    rc = lib.attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, scale,
                         int(bool(causal)), dt, _ptr(q_descale), _ptr(k_descale), _ptr(v_descale),
                         _ptr(workspace), 0 if workspace is None else workspace.numel() * workspace.element_size(),
                         _stream(stream))
    _check(rc, "attn_fwd")
    return out, lse


def quantize_e4m3(x, rmsnorm=False, eps=1e-6, codes=None, descale=None, stream=None):
    """bf16 x [B,H,S,D] -> (e4m3fn codes [B,H,S,D], fp32 descale [B,H]) with an
    optional per-row RMS normalisation first (see attn_quantize_e4m3 in hattn.h)."""
    _require(x, "x")
    if x.dtype != torch.bfloat16 or x.dim() != 4:
        raise TypeError("quantize_e4m3 takes a [B,H,S,D] bfloat16 tensor")
    B, H, S, D = x.shape
    if codes is None:
        codes = torch.empty((B, H, S, D), dtype=torch.float8_e4m3fn, device=x.device)
    if descale is None:
        descale = torch.empty((B, H), dtype=torch.float32, device=x.device)
    rc = lib.attn_quantize_e4m3(_ptr(x), _ptr(codes), _ptr(descale), B, H, S, D, int(bool(rmsnorm)), float(eps),
                                _stream(stream))
    _check(rc, "attn_quantize_e4m3")
    return codes, descale


def kvblocks_workspace_size(B, Hq, Sq, D, n_blocks) -> int:
    return lib.attn_fwd_kvblocks_workspace_size(B, Hq, Sq, D, n_blocks)


def attn_fwd_kvblocks(q, k_blocks, v_blocks, scale=None, workspace=None, out=None, lse=None, stream=None):
    """Unmasked attention of q to the concatenation of the KV blocks, per block + fixed-order LSE merge."""
    _require(q, "q")
    n = len(k_blocks)
    if n != len(v_blocks) or n == 0:
        raise ValueError("need the same non-zero number of K and V blocks")
    for t in list(k_blocks) + list(v_blocks):
        _require(t, "kv block")
    B, Hq, Sq, D = q.shape
    Hkv = k_blocks[0].shape[1]
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    kp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in k_blocks])
    vp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in v_blocks])
    lens = (ctypes.c_int * n)(*[int(t.shape[2]) for t in k_blocks])
    ws_bytes = kvblocks_workspace_size(B, Hq, Sq, D, n)
    if workspace is None and ws_bytes:
        workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=q.device)
    if out is None:
        out = torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=q.device)
    if lse is None:
        lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=q.device)
    rc = lib.attn_fwd_kvblocks(_ptr(q), ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                               ctypes.cast(lens, ctypes.c_void_p), n, _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, D,
                               scale, _dtype_code(q), None, None, None, _ptr(workspace),
                               0 if workspace is None else workspace.numel() * workspace.element_size(),
                               _stream(stream))
    _check(rc, "attn_fwd_kvblocks")
    return out, lse


def bwd_workspace_size(B, Hq, Sq) -> int:
    return lib.attn_bwd_workspace_size(B, Hq, Sq)


def attn_bwd(q, k, v, out, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
             stream=None):
    """dQ, dK, dV (bf16) of attention for upstream gradient dout."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (lse, "lse"), (dout, "dout")):
        _require(t, n)
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    if workspace is None:
        workspace = torch.empty(bwd_workspace_size(B, Hq, Sq), dtype=torch.uint8, device=q.device)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    rc = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk), _ptr(dv),
                      B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), _ptr(workspace),
                      workspace.numel() * workspace.element_size(), _stream(stream))
    _check(rc, "attn_bwd")
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, out, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None, stream=None):
    """attn_bwd without a workspace, for callers that may not allocate device
    scratch; the library's static 16 MiB array holds Delta (B*Hq*Sq <= 2^22)."""
    for t, n in ((q, "q"), (k, "k"), (v, "v"), (out, "out"), (lse, "lse"), (dout, "dout")):
        _require(t, n)
    B, Hq, Sq, D = q.shape
    _, Hkv, Sk, _ = k.shape
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    dq = torch.empty_like(q) if dq is None else dq
    dk = torch.empty_like(k) if dk is None else dk
    dv = torch.empty_like(v) if dv is None else dv
    rc = lib.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                              _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), _stream(stream))
    _check(rc, "attn_bwd_noalloc")
    return dq, dk, dv


def get_device_error(stream=None) -> int:
    """Synchronise and read-and-clear the kernels' bounded-wait error word (0 = none)."""
    code = ctypes.c_int(0)
    _check(lib.attn_get_device_error(_stream(stream), ctypes.byref(code)), "attn_get_device_error")
    return code.value
