"""B200 (sm_100a) fused scaled-dot-product attention: forward (bf16 / e4m3 with
descales, with LSE), block-KV streaming forward with a fixed-order LSE merge,
a context-parallel forward over torch.distributed ranks built on it, and a
deterministic backward.  The kernels live in libhattn.so (built from
csrc/ by build.py); this package is its ctypes binding.

The binding is loaded on first use of any of its names, so ``build`` can be
imported before the library exists; using the API without the library raises
ImportError (there is no fallback).

Usage (contiguous CUDA tensors [B, H, S, 128]; calls run on the tensors'
device and its current stream, allocate outputs unless given, and raise
HattnError with the library's code for a request it refuses)::

    import head_attention_qk_b200 as hattn
    out, lse = hattn.attn_fwd(q, k, v, causal=True)             # bf16 -> bf16 O, fp32 LSE
    dq, dk, dv = hattn.attn_bwd(q, k, v, out, lse, dout, causal=True)
    qc, qd = hattn.quantize_e4m3(q, rmsnorm=True)                # e4m3 codes + per-head descales
    kc, kd = hattn.quantize_e4m3(k, rmsnorm=True)
    vc, vd = hattn.quantize_e4m3(v)
    out8, lse8 = hattn.attn_fwd(qc, kc, vc, q_descale=qd, k_descale=kd, v_descale=vd)
    out_s, lse_s = hattn.attn_fwd_kvblocks(q, [k0, k1, k2], [v0, v1, v2])   # blocks folded in order
"""
_API = ("BF16", "E4M3", "EXPORTED", "NOALLOC_MAX_ROWS", "HattnError", "attn_bwd", "attn_bwd_noalloc",
        "attn_bwd_onepass", "bwd_onepass_workspace_size", "attn_bwd_dsbuf", "bwd_dsbuf_workspace_size", "attn_fwd",
        "attn_fwd_kvblocks", "bwd_workspace_size", "fwd_workspace_size", "get_device_error", "kvblocks_workspace_size",
        "lib", "quantize_e4m3")


_CP_API = ("attn_fwd_context_parallel", "gather_kv_shards")


def __getattr__(name):
    if name in _API:
        from . import hattn

        return getattr(hattn, name)
    if name in _CP_API:
        from . import context_parallel

        return getattr(context_parallel, name)
    raise AttributeError(name)


def __dir__():
    return sorted(list(globals()) + list(_API) + list(_CP_API))
