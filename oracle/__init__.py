"""CPU fp64 attention oracle -- test infrastructure only (see oracle.py)."""
from .oracle import (attn_bwd, attn_fwd, build, build_mutant, e4m3_rne, e4m3_to_double, lse_merge, num_threads,  # noqa: F401
                     quantize_e4m3)
