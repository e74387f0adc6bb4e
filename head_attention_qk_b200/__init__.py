"""B200 (sm_100a) fused scaled-dot-product attention: forward (bf16 / e4m3 with
descales, with LSE), block-KV streaming forward with a fixed-order LSE merge,
and a deterministic backward.  The kernels live in libhattn.so (built from
csrc/ by build.py); this package is its ctypes binding.
"""
from .hattn import (  # noqa: F401
    BF16,
    E4M3,
    EXPORTED,
    HattnError,
    attn_bwd,
    attn_fwd,
    attn_fwd_kvblocks,
    bwd_workspace_size,
    get_device_error,
    kvblocks_workspace_size,
    lib,
)
