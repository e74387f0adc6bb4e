"""The five workloads the library is sized and measured for.

Shapes follow the pages' workloads:
- tiny: a small self-attention the oracle finishes in seconds;
- llm_gqa: Qwen3-8B dense heads (Hq=32, Hkv=8, D=128), causal prefill, bf16,
  forward and backward (RL-Kernel PR #319, ROCm Validation and Benchmark
  results tables, B=2/4 at S=2048);
- video: a video-DiT self-attention over 21 latent frames of 30x52 tokens with
  per-head Q/K normalisation (FlashDreams PR #486, section 1.2, "head- or
  inner-scoped Q/K normalization"); 40 heads as in the Wan 14B blocks
  (AITER PR #2911, Wan 2.2 cross-attention repro with -n 40);
- fp8: the AITER fp8 fmha benchmark shape b=1, n=5, q=75600, d=128
  (AITER PR #2911, Test Result), e4m3fn with per-head descales;
- streaming: new-frame queries (one frame chunk of 1560 tokens) against a
  block KV cache of 21 blocks, plus cross-attention to 512 text tokens
  (FlashDreams PR #486, section 1.2: streaming self-attention over a block KV
  cache and static cross-attention).

Two more shapes from the pages' streaming workloads, measured beside these:
- cross: long-query cross-attention, Sq=90000 video tokens against Sk=512 text
  tokens with 40 heads (AITER PR #2911, the Wan 2.2 cross-attention report);
- window: the raw SDPA call on the window-30 shape, 4680 queries against 51480
  keys with 12 heads (FlashDreams issue #739, "SDPA kernels on gfx950").
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    Hq: int
    Hkv: int
    Sq: int
    Sk: int
    D: int = 128
    causal: bool = False
    dtype: str = "bf16"          # "bf16" or "e4m3"
    seed: int = 0
    qk_rmsnorm: bool = False
    backward: bool = False
    n_blocks: int = 0            # streaming: number of KV-cache blocks of length Sk // n_blocks
    text_len: int = 0            # streaming: cross-attention key length
    per_row_seed: bool = False   # llm_gqa: each batch row drawn from seed + b
    extra: dict = field(default_factory=dict)

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)

    def fwd_flops(self) -> float:
        """4 B Hq Sq Sk D, halved for causal (AITER PR #2911, Test Result:
        4*1*5*75600^2*128 flop / 7082.7 us = 2065.8 TFLOPS as printed)."""
        f = 4.0 * self.B * self.Hq * self.Sq * self.Sk * self.D
        return f / 2 if self.causal else f

    def bwd_flops(self) -> float:
        """Conventional backward count: 2.5x the forward."""
        return 2.5 * self.fwd_flops()


CONFIGS = {
    "tiny": Workload("tiny", B=1, Hq=2, Hkv=2, Sq=256, Sk=256, seed=0),
    "llm_gqa": Workload("llm_gqa", B=2, Hq=32, Hkv=8, Sq=2048, Sk=2048, causal=True, seed=1000,
                        backward=True, per_row_seed=True),
    "video": Workload("video", B=1, Hq=40, Hkv=40, Sq=32760, Sk=32760, seed=2, qk_rmsnorm=True),
    "fp8": Workload("fp8", B=1, Hq=5, Hkv=5, Sq=75600, Sk=75600, dtype="e4m3", seed=3),
    "streaming": Workload("streaming", B=1, Hq=40, Hkv=40, Sq=1560, Sk=21 * 1560, seed=4,
                          n_blocks=21, text_len=512),
    "cross": Workload("cross", B=1, Hq=40, Hkv=40, Sq=90000, Sk=512, seed=5),
    "window": Workload("window", B=1, Hq=12, Hkv=12, Sq=4680, Sk=51480, seed=6),
    # the precision pair the FP8 page compares (AITER PR #2911, Test Result:
    # bf16 and fp8 fmha on the same 75600-token shape), measured on both shapes
    "bf16_75600": Workload("bf16_75600", B=1, Hq=5, Hkv=5, Sq=75600, Sk=75600, seed=7),
    "fp8_32760": Workload("fp8_32760", B=1, Hq=40, Hkv=40, Sq=32760, Sk=32760, dtype="e4m3", seed=8,
                          qk_rmsnorm=True),
}


def get(name: str, **overrides) -> Workload:
    w = CONFIGS[name]
    if overrides:
        d = dict(w.__dict__)
        d.update(overrides)
        w = Workload(**d)
    return w
