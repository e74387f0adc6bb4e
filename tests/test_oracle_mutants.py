"""The oracle's pins catch plausible mistakes.

Each entry of MUTANTS plants one mistake in the oracle (a dropped term, a
wrong sign, index or operand, a wrong constant or rounding rule), compiled
in with -DORACLE_MUTANT=n, and runs the CPU pin suites against that build.
Every one of them must make a pin fail (pytest exit status 1: a failed
assertion, not a crash).  Mistakes are planted in the oracle only, on the
CPU; the GPU library is not involved.
"""
import os
import subprocess
import sys

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_invariants.py", "tests/test_oracle_prologue.py"]

MUTANTS = {
    1: "scores without the softmax scale",
    2: "causal mask aligned top-left instead of bottom-right",
    3: "query head h reads KV head h % Hkv instead of h / (Hq / Hkv)",
    4: "LSE without the row maximum added back",
    5: "probabilities normalised by the row maximum instead of the LSE",
    6: "K read transposed (d-major)",
    7: "v_descale not applied",
    8: "merge weight of a block taken from the running LSE",
    9: "merged LSE without the maximum added back",
    10: "dS = P (Delta - dP): sign flipped",
    11: "dK without the scale",
    12: "dV accumulates dS instead of P",
    13: "Delta formed from q instead of O",
    14: "dK and dV from the first query head of each group only",
    15: "descale = amax / 447",
    16: "e4m3 rounding with ties to the odd code",
    17: "RMS norm without eps",
    18: "e4m3 subnormals decoded at 2^-7 instead of 2^-6",
    19: "bf16 widened with a 15-bit shift",
    20: "causal mask one key short (j < i + Sk - Sq)",
    21: "head maximum taken before the RMS norm",
    22: "RMS mean over 127 instead of 128",
    25: "backward without the causal mask",
    27: "dQ without the scale",
    29: "e4m3 NaN code decoded as 480",
    30: "q_descale indexed by the KV head",
    31: "merged O not divided by the sum of the weights",
    32: "negative values that round to zero lose their sign bit",
    34: "sampled query rows ignored (row r evaluated instead of rows[r])",
    36: "Delta over the first half of the head dimension only",
    41: "head maximum skips the last row",
    42: "RMS factor 1 / (sqrt(mean) + eps) instead of 1 / sqrt(mean + eps)",
    47: "backward groups query heads kv + g * Hkv instead of kv * G + g",
}


def test_every_planted_mistake_fails_a_pin():
    normal = oracle.build()
    out_dir = os.path.join(ROOT, "oracle", ".mutants")
    os.makedirs(out_dir, exist_ok=True)
    libs = {n: oracle.build_mutant(n, os.path.join(out_dir, "liboracle_m%d.so" % n)) for n in MUTANTS}
    try:
        results = {}
        libs[0] = normal                 # control: the same run on the normal build must pass
        pending = [0] + list(MUTANTS)
        running = {}
        while pending or running:
            while pending and len(running) < 6:
                n = pending.pop(0)
                env = dict(os.environ, ORACLE_LIB=libs[n], OMP_NUM_THREADS="2")
                cmd = [sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *PIN_FILES]
                running[n] = subprocess.Popen(cmd, cwd=ROOT, env=env, stdout=subprocess.DEVNULL,
                                              stderr=subprocess.DEVNULL)
            for n, p in list(running.items()):
                if p.poll() is not None:
                    results[n] = p.returncode
                    del running[n]
            if running:
                next(iter(running.values())).wait(timeout=600)
        assert results.pop(0) == 0, "the pin suites fail on the normal build when run this way"
        survivors = {n: (MUTANTS[n], rc) for n, rc in results.items() if rc != 1}
        assert not survivors, "planted mistakes that no pin caught (mutant: (what, pytest status)): %s" % survivors
    finally:
        for n, path in libs.items():
            if n and os.path.exists(path):
                os.remove(path)
        if not os.listdir(out_dir):
            os.rmdir(out_dir)
