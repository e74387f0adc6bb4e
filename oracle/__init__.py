"""CPU fp64 attention oracle -- test infrastructure only (see oracle.py)."""
from .oracle import (attn_bwd, attn_fwd, build, compile_library, e4m3_rne, e4m3_to_double, lse_merge, num_threads, source_path,  # noqa: F401
                     quantize_e4m3)
