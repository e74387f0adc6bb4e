"""Seeded synthetic workloads for the attention library and its oracle.

This package only draws inputs (and applies the input preparation the
workloads call for: per-head RMS normalisation of Q/K, e4m3 quantisation with
per-head descales).  It holds none of the attention arithmetic, and it imports
neither the CUDA library nor the oracle, so both sides can take their inputs
from it.
"""
from .configs import CONFIGS, Workload, get  # noqa: F401
from .gen import (  # noqa: F401
    bf16_bits,
    e4m3_bits,
    make_bwd_inputs,
    make_fwd_inputs,
    make_kvblock_inputs,
    quantize_e4m3_per_head,
    rms_normalize,
    sample_rows,
)
