"""The FLOP convention of the benchmark, pinned to numbers the pages print.

AITER PR #2911 ("F8 fmha ASM gfx950", Test Result) prints both the kernel time
and the TFLOPS it derives; the forward count 4*B*H*Sq*Sk*D must reproduce the
printed TFLOPS from the printed time.
"""
import os

import pytest

from workloads import Workload

HERE = os.path.dirname(os.path.abspath(__file__))


def rows():
    with open(os.path.join(HERE, "golden", "aiter_fmha_mi355x.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                yield line.split()


@pytest.mark.parametrize("row", list(rows()), ids=lambda r: r[0])
def test_fwd_flop_convention_reproduces_printed_tflops(row):
    name, B, H, Sq, Sk, D, causal, t_us, tflops = row
    w = Workload(name, B=int(B), Hq=int(H), Hkv=int(H), Sq=int(Sq), Sk=int(Sk), D=int(D), causal=bool(int(causal)))
    got = w.fwd_flops() / (float(t_us) * 1e-6) / 1e12
    assert abs(got - float(tflops)) / float(tflops) < 1e-6, (got, tflops)


def test_causal_halves_the_count():
    a = Workload("a", B=2, Hq=32, Hkv=8, Sq=2048, Sk=2048, causal=False)
    b = Workload("b", B=2, Hq=32, Hkv=8, Sq=2048, Sk=2048, causal=True)
    assert b.fwd_flops() * 2 == a.fwd_flops()
    assert b.bwd_flops() == 2.5 * b.fwd_flops()
