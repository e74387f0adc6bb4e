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
lib.attn_bwd_dsbuf.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz,
                               _vp]
lib.attn_bwd_dsbuf.restype = _i
lib.attn_bwd_dsbuf_workspace_size.argtypes = [_i, _i, _i, _i]
lib.attn_bwd_dsbuf_workspace_size.restype = _sz
lib.attn_bwd_onepass.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _f, _i, _vp, _sz,
                                 _vp]
lib.attn_bwd_onepass.restype = _i
lib.attn_bwd_onepass_workspace_size.argtypes = [_i, _i, _i]
lib.attn_bwd_onepass_workspace_size.restype = _sz
lib.attn_selftest_counter_wait.argtypes = [_vp, _vp, ctypes.c_uint]
lib.attn_selftest_counter_wait.restype = _i
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
            "attn_bwd_workspace_size", "attn_bwd_dsbuf", "attn_bwd_dsbuf_workspace_size", "attn_bwd_onepass", "attn_bwd_onepass_workspace_size", "attn_bwd_noalloc",
            "attn_get_device_error", "attn_selftest_bounded_wait", "attn_selftest_counter_wait", "attn_error_string")
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


# Argument checks.  The library sees only pointers and the sizes passed with
# them, so every tensor's shape and dtype are checked against those sizes here
# (a buffer smaller than the sizes say would be read or written out of
# bounds).  Shapes and dtypes are checked first, then that every tensor is a
# contiguous CUDA tensor on one device; the call runs with that device current
# and, by default, on its current stream.  Outputs and scratch the binding
# allocates are taken from torch's caching allocator while the launch stream
# is torch's current stream, so the allocator never hands them to work on
# another stream while the kernels may still use them (scratch is released
# on return, and its next owner is ordered after the kernels on that stream).

def _shape(t, name, shape):
    if not isinstance(t, torch.Tensor):
        raise TypeError("%s must be a torch.Tensor" % name)
    if tuple(t.shape) != tuple(shape):
        raise ValueError("%s must have shape %s, got %s" % (name, tuple(shape), tuple(t.shape)))


def _dtype(t, name, *dtypes):
    if t.dtype not in dtypes:
        raise TypeError("%s must be %s, got %s" % (name, " or ".join(str(d) for d in dtypes), t.dtype))


def _dims4(t, name):
    if not isinstance(t, torch.Tensor) or t.dim() != 4:
        raise ValueError("%s must be a 4-d [B, H, S, D] tensor" % name)
    return tuple(int(x) for x in t.shape)


def _device(named):
    """The one CUDA device of the (name, tensor) pairs (None entries skipped)."""
    dev = None
    for name, t in named:
        if t is None:
            continue
        if not t.is_cuda:
            raise ValueError("%s must be a CUDA tensor" % name)
        if not t.is_contiguous():
            raise ValueError("%s must be contiguous" % name)
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError("%s is on %s, the other tensors on %s" % (name, t.device, dev))
    return dev


def _stream(stream, dev=None):
    """The torch stream a call runs on: `stream`, else the device's current stream."""
    if stream is None:
        stream = torch.cuda.current_stream(dev)
    elif dev is not None and stream.device != dev:
        raise ValueError("stream is on %s, the tensors on %s" % (stream.device, dev))
    return stream


def _sp(stream):
    return ctypes.c_void_p(stream.cuda_stream)


def _nbytes(t):
    return 0 if t is None else t.numel() * t.element_size()


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return BF16
    if t.dtype == torch.float8_e4m3fn:
        return E4M3
    raise TypeError("inputs must be bfloat16 or float8_e4m3fn, got %s" % t.dtype)


def _descales(B, Hq, Hkv, q_descale, k_descale, v_descale):
    """Size and type of each descale given; which ones must be given (all three
    for e4m3, none for bf16) is the library's check (HATTN_EINVAL)."""
    for d, name, n in ((q_descale, "q_descale", B * Hq), (k_descale, "k_descale", B * Hkv),
                       (v_descale, "v_descale", B * Hkv)):
        if d is None:
            continue
        _dtype(d, name, torch.float32)
        if d.numel() != n:
            raise ValueError("%s must hold %d values (one per batch and head), got %d" % (name, n, d.numel()))


def fwd_workspace_size(B, Hkv, Sk, D, dtype) -> int:
    return lib.attn_fwd_workspace_size(B, Hkv, Sk, D, dtype)


def attn_fwd(q, k, v, causal=False, scale=None, q_descale=None, k_descale=None, v_descale=None,
             out=None, lse=None, workspace=None, stream=None, use_scratch=True):
    """O [B,Hq,Sq,D] bf16 and LSE [B,Hq,Sq] fp32 for q [B,Hq,Sq,D], k/v [B,Hkv,Sk,D].

    e4m3 inputs take scratch for the fp16 copy of V (the faster of the
    library's two e4m3 forms, same results): `workspace` (a CUDA byte tensor of
    at least fwd_workspace_size() bytes), else one from torch's allocator.
    With use_scratch=False the call takes none and the library widens V in
    shared memory (attn_fwd of the C ABI).
    """
    B, Hq, Sq, D = _dims4(q, "q")
    _, Hkv, Sk, _ = _dims4(k, "k")
    _shape(k, "k", (B, Hkv, Sk, D))
    _shape(v, "v", (B, Hkv, Sk, D))
    dt = _dtype_code(q)
    _dtype(k, "k", q.dtype)
    _dtype(v, "v", q.dtype)
    _descales(B, Hq, Hkv, q_descale, k_descale, v_descale)
    if out is not None:
        _shape(out, "out", (B, Hq, Sq, D))
        _dtype(out, "out", torch.bfloat16)
    if lse is not None:
        _shape(lse, "lse", (B, Hq, Sq))
        _dtype(lse, "lse", torch.float32)
    dev = _device([("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("q_descale", q_descale),
                   ("k_descale", k_descale), ("v_descale", v_descale), ("workspace", workspace)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if out is None:
            out = torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
        if not use_scratch:
            if workspace is not None:
                raise ValueError("workspace given with use_scratch=False")
            rc = lib.attn_fwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, scale,
                              int(bool(causal)), dt, _ptr(q_descale), _ptr(k_descale), _ptr(v_descale), _sp(st))
        else:
            ws_bytes = fwd_workspace_size(B, Hkv, Sk, D, dt)
            if ws_bytes and workspace is None:
                workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
            rc = lib.attn_fwd_ws(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, Sk, D, scale,
                                 int(bool(causal)), dt, _ptr(q_descale), _ptr(k_descale), _ptr(v_descale),
                                 _ptr(workspace), _nbytes(workspace), _sp(st))
    _check(rc, "attn_fwd")
    return out, lse


def quantize_e4m3(x, rmsnorm=False, eps=1e-6, codes=None, descale=None, stream=None):
    """bf16 x [B,H,S,D] -> (e4m3fn codes [B,H,S,D], fp32 descale [B,H]) with an
    optional per-row RMS normalisation first (see attn_quantize_e4m3 in hattn.h)."""
    B, H, S, D = _dims4(x, "x")
    _dtype(x, "x", torch.bfloat16)
    if codes is not None:
        _shape(codes, "codes", (B, H, S, D))
        _dtype(codes, "codes", torch.float8_e4m3fn)
    if descale is not None:
        _dtype(descale, "descale", torch.float32)
        if descale.numel() != B * H:
            raise ValueError("descale must hold %d values (one per batch and head)" % (B * H))
    dev = _device([("x", x), ("codes", codes), ("descale", descale)])
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if codes is None:
            codes = torch.empty((B, H, S, D), dtype=torch.float8_e4m3fn, device=dev)
        if descale is None:
            descale = torch.empty((B, H), dtype=torch.float32, device=dev)
        rc = lib.attn_quantize_e4m3(_ptr(x), _ptr(codes), _ptr(descale), B, H, S, D, int(bool(rmsnorm)),
                                    float(eps), _sp(st))
    _check(rc, "attn_quantize_e4m3")
    return codes, descale


def kvblocks_workspace_size(B, Hq, Sq, D, n_blocks) -> int:
    return lib.attn_fwd_kvblocks_workspace_size(B, Hq, Sq, D, n_blocks)


def attn_fwd_kvblocks(q, k_blocks, v_blocks, scale=None, workspace=None, out=None, lse=None, stream=None,
                      q_descale=None, k_descale=None, v_descale=None):
    """Unmasked attention of q to the concatenation of the KV blocks, folded in block order.

    e4m3 blocks (an FP8 KV cache) take q_descale [B, Hq] and k_descale,
    v_descale [n_blocks, B, Hkv] (one scale per block and head; any shape with
    that many fp32 values, block-major)."""
    B, Hq, Sq, D = _dims4(q, "q")
    n = len(k_blocks)
    if n != len(v_blocks) or n == 0:
        raise ValueError("need the same non-zero number of K and V blocks")
    dt = _dtype_code(q)
    Hkv = _dims4(k_blocks[0], "k_blocks[0]")[1]
    lens = []
    for i, (kb, vb) in enumerate(zip(k_blocks, v_blocks)):
        L = _dims4(kb, "k_blocks[%d]" % i)[2]
        _shape(kb, "k_blocks[%d]" % i, (B, Hkv, L, D))
        _shape(vb, "v_blocks[%d]" % i, (B, Hkv, L, D))
        _dtype(kb, "k_blocks[%d]" % i, q.dtype)
        _dtype(vb, "v_blocks[%d]" % i, q.dtype)
        lens.append(L)
    for d, name, cnt in ((q_descale, "q_descale", B * Hq), (k_descale, "k_descale", n * B * Hkv),
                         (v_descale, "v_descale", n * B * Hkv)):
        if d is not None:
            _dtype(d, name, torch.float32)
            if d.numel() != cnt:
                raise ValueError("%s must hold %d values, got %d" % (name, cnt, d.numel()))
    if out is not None:
        _shape(out, "out", (B, Hq, Sq, D))
        _dtype(out, "out", torch.bfloat16)
    if lse is not None:
        _shape(lse, "lse", (B, Hq, Sq))
        _dtype(lse, "lse", torch.float32)
    dev = _device([("q", q), ("out", out), ("lse", lse), ("workspace", workspace), ("q_descale", q_descale),
                   ("k_descale", k_descale), ("v_descale", v_descale)]
                  + [("k_blocks[%d]" % i, t) for i, t in enumerate(k_blocks)]
                  + [("v_blocks[%d]" % i, t) for i, t in enumerate(v_blocks)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    kp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in k_blocks])
    vp = (ctypes.c_void_p * n)(*[t.data_ptr() for t in v_blocks])
    ln = (ctypes.c_int * n)(*lens)
    ws_bytes = kvblocks_workspace_size(B, Hq, Sq, D, n)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if workspace is None and ws_bytes:
            workspace = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
        if out is None:
            out = torch.empty((B, Hq, Sq, D), dtype=torch.bfloat16, device=dev)
        if lse is None:
            lse = torch.empty((B, Hq, Sq), dtype=torch.float32, device=dev)
        rc = lib.attn_fwd_kvblocks(_ptr(q), ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(vp, ctypes.c_void_p),
                                   ctypes.cast(ln, ctypes.c_void_p), n, _ptr(out), _ptr(lse), B, Hq, Hkv, Sq, D,
                                   scale, dt, _ptr(q_descale), _ptr(k_descale), _ptr(v_descale), _ptr(workspace),
                                   _nbytes(workspace), _sp(st))
    _check(rc, "attn_fwd_kvblocks")
    return out, lse


def bwd_workspace_size(B, Hq, Sq) -> int:
    return lib.attn_bwd_workspace_size(B, Hq, Sq)


def _bwd_args(q, k, v, out, lse, dout, dq, dk, dv):
    """Sizes of a backward call after checking every tensor against them."""
    B, Hq, Sq, D = _dims4(q, "q")
    _, Hkv, Sk, _ = _dims4(k, "k")
    for t, name, shape in ((k, "k", (B, Hkv, Sk, D)), (v, "v", (B, Hkv, Sk, D)), (out, "out", (B, Hq, Sq, D)),
                           (dout, "dout", (B, Hq, Sq, D)), (dq, "dq", (B, Hq, Sq, D)), (dk, "dk", (B, Hkv, Sk, D)),
                           (dv, "dv", (B, Hkv, Sk, D))):
        if t is not None:
            _shape(t, name, shape)
            _dtype(t, name, torch.bfloat16)
    _dtype(q, "q", torch.bfloat16)
    _shape(lse, "lse", (B, Hq, Sq))
    _dtype(lse, "lse", torch.float32)
    return B, Hq, Hkv, Sq, Sk, D


def attn_bwd(q, k, v, out, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
             stream=None):
    """dQ, dK, dV (bf16) of attention for upstream gradient dout."""
    B, Hq, Hkv, Sq, Sk, D = _bwd_args(q, k, v, out, lse, dout, dq, dk, dv)
    dev = _device([("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout), ("dq", dq),
                   ("dk", dk), ("dv", dv), ("workspace", workspace)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if workspace is None:
            workspace = torch.empty(bwd_workspace_size(B, Hq, Sq), dtype=torch.uint8, device=dev)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        rc = lib.attn_bwd(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                          _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), _ptr(workspace),
                          _nbytes(workspace), _sp(st))
    _check(rc, "attn_bwd")
    return dq, dk, dv


def bwd_dsbuf_workspace_size(B, Hq, Sq, Sk) -> int:
    return lib.attn_bwd_dsbuf_workspace_size(B, Hq, Sq, Sk)


def attn_bwd_dsbuf(q, k, v, out, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
                   stream=None):
    """dQ, dK, dV (bf16) with dS stored in the workspace (O(Sq x Sk) bytes,
    see bwd_dsbuf_workspace_size): dQ is read back as the product dS K."""
    B, Hq, Hkv, Sq, Sk, D = _bwd_args(q, k, v, out, lse, dout, dq, dk, dv)
    dev = _device([("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout), ("dq", dq),
                   ("dk", dk), ("dv", dv), ("workspace", workspace)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if workspace is None:
            workspace = torch.empty(bwd_dsbuf_workspace_size(B, Hq, Sq, Sk), dtype=torch.uint8, device=dev)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        rc = lib.attn_bwd_dsbuf(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), _ptr(workspace),
                                _nbytes(workspace), _sp(st))
    _check(rc, "attn_bwd_dsbuf")
    return dq, dk, dv


def bwd_onepass_workspace_size(B, Hq, Sq) -> int:
    return lib.attn_bwd_onepass_workspace_size(B, Hq, Sq)


def attn_bwd_onepass(q, k, v, out, lse, dout, causal=False, scale=None, workspace=None, dq=None, dk=None, dv=None,
                     stream=None):
    """dQ, dK, dV (bf16) from the one-pass backward (one kernel, dQ added in
    key-tile order through an fp32 accumulator in the workspace)."""
    B, Hq, Hkv, Sq, Sk, D = _bwd_args(q, k, v, out, lse, dout, dq, dk, dv)
    dev = _device([("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout), ("dq", dq),
                   ("dk", dk), ("dv", dv), ("workspace", workspace)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        if workspace is None:
            workspace = torch.empty(bwd_onepass_workspace_size(B, Hq, Sq), dtype=torch.uint8, device=dev)
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        rc = lib.attn_bwd_onepass(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq), _ptr(dk),
                                  _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)), _ptr(workspace),
                                  _nbytes(workspace), _sp(st))
    _check(rc, "attn_bwd_onepass")
    return dq, dk, dv


def attn_bwd_noalloc(q, k, v, out, lse, dout, causal=False, scale=None, dq=None, dk=None, dv=None, stream=None):
    """attn_bwd without a workspace, for callers that may not allocate device
    scratch; the library's static 16 MiB array holds Delta (B*Hq*Sq <= 2^22)."""
    B, Hq, Hkv, Sq, Sk, D = _bwd_args(q, k, v, out, lse, dout, dq, dk, dv)
    dev = _device([("q", q), ("k", k), ("v", v), ("out", out), ("lse", lse), ("dout", dout), ("dq", dq),
                   ("dk", dk), ("dv", dv)])
    scale = 1.0 / math.sqrt(D) if scale is None else float(scale)
    st = _stream(stream, dev)
    with torch.cuda.device(dev), torch.cuda.stream(st):
        dq = torch.empty_like(q) if dq is None else dq
        dk = torch.empty_like(k) if dk is None else dk
        dv = torch.empty_like(v) if dv is None else dv
        rc = lib.attn_bwd_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(out), _ptr(lse), _ptr(dout), _ptr(dq),
                                  _ptr(dk), _ptr(dv), B, Hq, Hkv, Sq, Sk, D, scale, int(bool(causal)),
                                  _sp(st))
    _check(rc, "attn_bwd_noalloc")
    return dq, dk, dv


def get_device_error(stream=None) -> int:
    """Synchronise and read-and-clear the kernels' bounded-wait error word (0 = none)."""
    code = ctypes.c_int(0)
    _check(lib.attn_get_device_error(_sp(_stream(stream)), ctypes.byref(code)), "attn_get_device_error")
    return code.value
