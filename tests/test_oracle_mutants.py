"""The oracle's pins catch plausible mistakes.

Each entry of MUTANTS plants one mistake in a copy of the oracle's C source
(a dropped term, a wrong sign, index or operand, a wrong constant or rounding
rule) as a text patch: the original snippet must occur exactly once in
oracle/attn_oracle.c, the patched copy is compiled into its own library, and
the CPU pin suites run against that build.  Every one of them must make a pin
fail (pytest exit status 1: a failed assertion, not a crash).  The oracle's
source itself carries none of this: it reads as the bare definition.
Mistakes are planted in the oracle only, on the CPU; the GPU library is not
involved.
"""
import os
import subprocess
import sys
import tempfile

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
PIN_FILES = ["tests/test_oracle_pins.py", "tests/test_oracle_invariants.py", "tests/test_oracle_prologue.py"]

_LAST = "int64_t last = i + ((int64_t)Sk - (int64_t)Sq);"
_RMS = "r = 1.0 / sqrt(ss / D + eps);"
_AMAX = "if (fabs(yv) > amax) amax = fabs(yv);"
_DELTA = "for (int d = 0; d < D; ++d) delta += dorow[d] * orow[d];"

# number: (what the mistake is, original snippet, replacement)
MUTANTS = {
    1: ("scores without the softmax scale", "s[j] = scale * acc;", "s[j] = acc;"),
    2: ("causal mask aligned top-left instead of bottom-right", _LAST, "int64_t last = i;"),
    3: ("query head h reads KV head h % Hkv instead of h / (Hq / Hkv)",
        "const int kh = h / G;", "const int kh = h % Hkv;"),
    4: ("LSE without the row maximum added back", "const double L = m + log(sum);", "const double L = log(sum);"),
    5: ("probabilities normalised by the row maximum instead of the LSE",
        "const double p = exp(s[j] - L);", "const double p = exp(s[j] - m);"),
    6: ("K read transposed (d-major)", "load_elem(kind, k, kvbase + j * D + d, dk)",
        "load_elem(kind, k, kvbase + d * (int64_t)Sk + j, dk)"),
    7: ("v_descale not applied", "const double dv = kind == ORACLE_E4M3 ? v_descale[(int64_t)b * Hkv + kh] : 1.0;",
        "const double dv = 1.0;"),
    8: ("merge weight of a block taken from the running LSE", "const double wb = exp(Lb - M);",
        "const double wb = exp(L - M);"),
    9: ("merged LSE without the maximum added back", "L = M + log(den);", "L = log(den);"),
    10: ("dS = P (Delta - dP): sign flipped", "const double ds = p[j] * (dp - delta);",
         "const double ds = p[j] * (delta - dp);"),
    11: ("dK without the scale", "dkh[j * D + d] += scale * ds * qrow[d];", "dkh[j * D + d] += ds * qrow[d];"),
    12: ("dV accumulates dS instead of P", "dvh[j * D + d] += p[j] * dorow[d];", "dvh[j * D + d] += ds * dorow[d];"),
    13: ("Delta formed from q instead of O", _DELTA, _DELTA.replace("orow[d];", "qrow[d];")),
    14: ("dK and dV from the first query head of each group only", "for (int g = 0; g < G; ++g) {",
         "for (int g = 0; g < 1; ++g) {"),
    15: ("descale = amax / 447", "(float)(amax / 448.0)", "(float)(amax / 447.0)"),
    16: ("e4m3 rounding with ties to the odd code", "((code + 1) & 1) == 0", "((code + 1) & 1) == 1"),
    17: ("RMS norm without eps", _RMS, "r = 1.0 / sqrt(ss / D);"),
    18: ("e4m3 subnormals decoded at 2^-7 instead of 2^-6", "mag = ldexp((double)m / 8.0, -6);",
         "mag = ldexp((double)m / 8.0, -7);"),
    19: ("bf16 widened with a 15-bit shift", "uint32_t u = ((uint32_t)bits) << 16;",
         "uint32_t u = ((uint32_t)bits) << 15;"),
    20: ("causal mask one key short (j < i + Sk - Sq)", _LAST, _LAST.replace(";", " - 1;")),
    21: ("head maximum taken before the RMS norm", _AMAX,
         "{ const double x0 = bf16_to_double(xh[s * D + d]); if (fabs(x0) > amax) amax = fabs(x0); }"),
    22: ("RMS mean over D - 1 instead of D", _RMS, "r = 1.0 / sqrt(ss / (D - 1) + eps);"),
    25: ("backward without the causal mask",
         "const int64_t last = last_visible_key(i, Sq, Sk, causal);\n                        if (last < 0) { lse[lidx]",
         "const int64_t last = last_visible_key(i, Sq, Sk, 0);\n                        if (last < 0) { lse[lidx]"),
    27: ("dQ without the scale", "dqrow[d] += scale * ds * load_elem", "dqrow[d] += ds * load_elem"),
    29: ("e4m3 NaN code decoded as 480", "if (e == 0xF && m == 0x7) return NAN;", "if (0) return NAN;"),
    30: ("q_descale indexed by the KV head", "q_descale[(int64_t)b * Hq + h]", "q_descale[(int64_t)b * Hkv + kh]"),
    31: ("merged O not divided by the sum of the weights", "orow[d] = (w * orow[d] + wb * ob[d]) / den;",
         "orow[d] = (w * orow[d] + wb * ob[d]);"),
    32: ("negative zero loses its sign bit", "const int neg = signbit(v) ? 1 : 0;", "const int neg = v < 0.0 ? 1 : 0;"),
    34: ("sampled query rows ignored (row r evaluated instead of rows[r])", "const int64_t i = rows ? rows[r] : r;",
         "const int64_t i = r;"),
    36: ("Delta over the first half of the head dimension only", _DELTA, _DELTA.replace("d < D;", "d < D / 2;")),
    41: ("head maximum skips the last row", _AMAX, "if (s < S - 1 && fabs(yv) > amax) amax = fabs(yv);"),
    42: ("RMS factor 1 / (sqrt(mean) + eps) instead of 1 / sqrt(mean + eps)", _RMS,
         "r = 1.0 / (sqrt(ss / D) + eps);"),
    47: ("backward groups query heads kv + g * Hkv instead of kv * G + g", "const int h = kh * G + g;",
         "const int h = kh + g * Hkv;"),
    48: ("RMS sum of squares over the first half of the row only",
         "for (int d = 0; d < D; ++d) {\n                    const double xv = bf16_to_double(xh[s * D + d]);",
         "for (int d = 0; d < D / 2; ++d) {\n                    const double xv = bf16_to_double(xh[s * D + d]);"),
    49: ("RMS factor applied twice (divides by the mean square)", _RMS, "r = 1.0 / (ss / D + eps);"),
}


def test_every_patch_applies_exactly_once():
    with open(oracle.source_path()) as f:
        src = f.read()
    missing = {n: what for n, (what, find, _) in MUTANTS.items() if src.count(find) != 1}
    assert not missing, "patches whose snippet does not occur exactly once in the oracle source: %s" % missing


def test_every_planted_mistake_fails_a_pin():
    normal = oracle.build()
    with open(oracle.source_path()) as f:
        src = f.read()
    with tempfile.TemporaryDirectory(prefix="oracle_mutants_") as tmp:
        libs = {0: normal}                   # control: the same run on the normal build must pass
        for n, (_, find, repl) in MUTANTS.items():
            assert src.count(find) == 1, n
            c_path = os.path.join(tmp, "attn_oracle_m%d.c" % n)
            with open(c_path, "w") as f:
                f.write(src.replace(find, repl))
            libs[n] = oracle.compile_library(c_path, os.path.join(tmp, "liboracle_m%d.so" % n))
        results = {}
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
    survivors = {n: (MUTANTS[n][0], rc) for n, rc in results.items() if rc != 1}
    assert not survivors, "planted mistakes that no pin caught (mutant: (what, pytest status)): %s" % survivors
