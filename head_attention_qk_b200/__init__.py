"""B200 (sm_100a) fused scaled-dot-product attention: forward (bf16 / e4m3 with
descales, with LSE), block-KV streaming forward with a fixed-order LSE merge,
a context-parallel forward over torch.distributed ranks built on it, and a
deterministic backward.  The kernels live in libhattn.so (built from
csrc/ by build.py); this package is its ctypes binding.

The binding is loaded on first use of any of its names, so ``build`` can be
imported before the library exists; using the API without the library raises
ImportError (there is no fallback).
"""
_API = ("BF16", "E4M3", "EXPORTED", "NOALLOC_MAX_ROWS", "HattnError", "attn_bwd", "attn_bwd_noalloc", "attn_fwd",
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
