"""The C ABI without a GPU: the library loads, exports every symbol hattn.h
declares, sizes its workspaces, and refuses bad requests on the host (fail
closed) before anything is launched."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def h():
    from head_attention_qk_b200 import build

    build.build()
    import head_attention_qk_b200 as pkg

    return pkg


def declared_symbols():
    txt = open(os.path.join(ROOT, "include", "hattn.h")).read()
    return sorted(set(re.findall(r"HATTN_API\s+[\w\s\*]+?\b(attn_\w+)\s*\(", txt)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    for s in ("attn_fwd", "attn_fwd_kvblocks", "attn_bwd", "attn_bwd_dsbuf", "attn_bwd_dsbuf_workspace_size",
              "attn_fwd_kvblocks_workspace_size",
              "attn_bwd_workspace_size", "attn_get_device_error", "attn_error_string"):
        assert s in syms


def test_library_exports_every_declared_symbol(h):
    for s in declared_symbols():
        assert hasattr(h.lib, s), s
        assert s in h.EXPORTED


def test_library_exports_nothing_undeclared(h):
    """The attn_* entry points in the library's dynamic symbol table are exactly
    those hattn.h declares (read with nm from the library built here)."""
    import shutil
    import subprocess

    nm = shutil.which("nm")
    if nm is None:
        pytest.skip("nm not available")
    from head_attention_qk_b200 import hattn

    out = subprocess.run([nm, "-D", "--defined-only", hattn.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = sorted({line.split()[-1] for line in out.splitlines() if line.split()[-1].startswith("attn_")})
    assert exported == declared_symbols()


def declared_signatures():
    """{name: [C parameter types]} of every HATTN_API function in hattn.h."""
    txt = open(os.path.join(ROOT, "include", "hattn.h")).read()
    txt = re.sub(r"/\*.*?\*/", " ", txt, flags=re.S)
    out = {}
    for m in re.finditer(r"HATTN_API\s+([\w\s\*]+?)\b(attn_\w+)\s*\(([^)]*)\)\s*;", txt):
        params = [" ".join(p.split()) for p in m.group(3).split(",") if p.strip() and p.strip() != "void"]
        out[m.group(2)] = (" ".join(m.group(1).split()), params)
    return out


def _ctype_of(decl):
    """The ctypes type of a C declaration "type name" ("ptr" for any pointer)."""
    import ctypes as C

    if "*" in decl:
        return "ptr"
    base = " ".join(w for w in decl.split()[:-1] if w != "const")    # drop the name
    table = {"int": C.c_int, "float": C.c_float, "double": C.c_double, "size_t": C.c_size_t,
             "unsigned int": C.c_uint}
    assert base in table, "unmapped C type: %r" % decl
    return table[base]


def test_binding_argtypes_match_the_header(h):
    """Every ctypes prototype in the binding has the header's parameter count and
    types (pointers as pointers, int/float/double/size_t/unsigned as such)."""
    import ctypes as C

    sigs = declared_signatures()
    assert set(sigs) == set(h.EXPORTED)
    for name, (ret, params) in sigs.items():
        fn = getattr(h.lib, name)
        assert len(fn.argtypes) == len(params), (name, fn.argtypes, params)
        for c_decl, ct in zip(params, fn.argtypes):
            want = _ctype_of(c_decl)
            if want == "ptr":
                assert ct in (C.c_void_p, C.c_char_p) or issubclass(ct, C._Pointer), (name, c_decl, ct)
            else:
                assert ct is want, (name, c_decl, ct)
        r = _ctype_of(ret + " result")
        if r == "ptr":
            assert fn.restype in (C.c_void_p, C.c_char_p), (name, ret, fn.restype)
        else:
            assert fn.restype is r, (name, ret, fn.restype)


def test_workspace_sizes(h):
    assert h.kvblocks_workspace_size(1, 40, 1560, 128, 21) == 0          # folded in one launch
    assert h.kvblocks_workspace_size(1, 40, 1560, 128, 40) == 40 * 40 * 1560 * 129 * 4
    assert h.bwd_workspace_size(2, 32, 2048) == 2 * 32 * 2048 * 4 + 256   # Delta, then the dQ unit counter
    assert h.bwd_workspace_size(1, 1, 3) == 256 + 256
    assert h.kvblocks_workspace_size(0, 1, 1, 128, 1) == 0


# Fake, never-dereferenced device addresses: every case below is refused by the
# host checks before any CUDA call.
A = ctypes.c_void_p(0x10000)
B_ = ctypes.c_void_p(0x20000)
MIS = ctypes.c_void_p(0x20008)


def fwd(h, q=A, k=A, v=A, out=A, lse=A, B=1, Hq=2, Hkv=2, Sq=128, Sk=128, D=128, scale=0.088, causal=0, dtype=0,
        qd=None, kd=None, vd=None):
    return h.lib.attn_fwd(q, k, v, out, lse, B, Hq, Hkv, Sq, Sk, D, scale, causal, dtype, qd, kd, vd, None)


@pytest.mark.parametrize("kw,code", [
    (dict(q=None), -1), (dict(lse=None), -1), (dict(B=0), -1), (dict(Sq=0), -1), (dict(Sk=-1), -1),
    (dict(Hq=3, Hkv=2), -1), (dict(scale=0.0), -1), (dict(scale=-1.0), -1), (dict(scale=float("nan")), -1),
    (dict(scale=float("inf")), -1),
    (dict(qd=A, kd=A, vd=A), -1),               # descales with bf16
    (dict(dtype=1), -1),                        # e4m3 without descales
    (dict(dtype=1, qd=A, kd=A, vd=None), -1),
    (dict(dtype=7), -1),
    (dict(D=64), -2), (dict(D=256), -2),        # only head dim 128
    (dict(causal=1, Sq=300, Sk=200), -2),       # causal rows without any key
    (dict(q=MIS), -3), (dict(out=MIS), -3), (dict(lse=MIS), -3),
])
def test_fwd_fails_closed(h, kw, code):
    assert fwd(h, **kw) == code


def test_fwd_workspace_size_and_checks(h):
    assert h.fwd_workspace_size(1, 5, 75600, 128, 1) == 5 * 75600 * 128 * 2    # e4m3: fp16 copy of V
    assert h.fwd_workspace_size(2, 8, 2048, 128, 0) == 0                       # bf16 needs none
    need = h.fwd_workspace_size(1, 2, 128, 128, 1)

    def call(ws=B_, wsb=need, dtype=1):
        d = A if dtype == 1 else None
        return h.lib.attn_fwd_ws(A, A, A, A, A, 1, 2, 2, 128, 128, 128, 0.088, 0, dtype, d, d, d, ws, wsb, None)

    assert call(wsb=need - 1) == -4
    assert call(ws=None) == -1
    assert call(ws=MIS) == -3


def test_quantize_fails_closed(h):
    def call(x=A, codes=B_, ds=A, B=1, H=2, S=64, D=128, rms=1, eps=1e-6):
        return h.lib.attn_quantize_e4m3(x, codes, ds, B, H, S, D, rms, eps, None)

    assert call(x=None) == -1 and call(ds=None) == -1 and call(S=0) == -1
    assert call(eps=0.0) == -1 and call(eps=-1.0) == -1     # rmsnorm needs eps > 0
    assert call(D=64) == -2
    assert call(x=MIS) == -3 and call(codes=MIS) == -3


def test_kvblocks_fails_closed(h):
    lib = h.lib

    def call(lens, n, ws=A, wsb=0, dtype=0, D=128, qd=None):
        kp = (ctypes.c_void_p * len(lens))(*([0x10000] * len(lens)))
        ln = (ctypes.c_int * len(lens))(*lens)
        return lib.attn_fwd_kvblocks(A, ctypes.cast(kp, ctypes.c_void_p), ctypes.cast(kp, ctypes.c_void_p),
                                     ctypes.cast(ln, ctypes.c_void_p), n, A, A, 1, 2, 2, 64, D, 0.088, dtype,
                                     qd, qd, qd, ws, wsb, None)

    assert call([100, 0], 2) == -2                       # a zero-length block
    assert call([100, 50], 0) == -1
    assert call([100, 50], 2, D=64) == -2
    assert call([100, 50], 2, dtype=1) == -1             # e4m3 blocks without descales
    assert call([100, 50], 2, dtype=0, qd=A) == -1       # descales given for bf16
    assert call([100, 50], 2, dtype=2, qd=A) == -1       # no such element type
    # more blocks than one launch folds: per-block partials need the workspace
    many = [40 + i for i in range(33)]
    need = h.kvblocks_workspace_size(1, 2, 64, 128, 33)
    assert need > 0 and h.kvblocks_workspace_size(1, 2, 64, 128, 32) == 0
    assert call(many, 33, wsb=need - 1) == -4            # workspace too small
    assert call(many, 33, ws=MIS, wsb=need) == -3
    assert call(many, 33, ws=None, wsb=need) == -1


def test_bwd_fails_closed(h):
    lib = h.lib
    need = h.bwd_workspace_size(1, 2, 128)

    def call(ws=A, wsb=need, causal=0, Sq=128, Sk=128, D=128, dq=A):
        return lib.attn_bwd(A, A, A, A, A, A, dq, A, A, 1, 2, 2, Sq, Sk, D, 0.088, causal, ws, wsb, None)

    assert call(wsb=need - 4) == -4
    assert call(wsb=1 * 2 * 128 * 4) == -4           # Delta alone: the dQ unit counter needs its bytes too
    assert call(dq=None) == -1
    assert call(dq=MIS) == -3
    assert call(D=96) == -2
    assert call(causal=1, Sq=256, Sk=128) == -2


def test_bwd_dsbuf_fails_closed(h):
    lib = h.lib
    need = h.bwd_dsbuf_workspace_size(1, 2, 128, 300)
    # Delta, then 2 heads x 3 key tiles x 1 query tile of 32 KB
    assert need >= 2 * 3 * 1 * 32768 + 2 * 128 * 4
    assert h.bwd_dsbuf_workspace_size(0, 2, 128, 300) == 0

    def call(ws=A, wsb=need, causal=0, Sq=128, Sk=300, D=128, dq=A):
        return lib.attn_bwd_dsbuf(A, A, A, A, A, A, dq, A, A, 1, 2, 2, Sq, Sk, D, 0.088, causal, ws, wsb, None)

    assert call(wsb=need - 1) == -4
    assert call(ws=None) == -1
    assert call(dq=None) == -1
    assert call(dq=MIS) == -3
    assert call(D=96) == -2
    assert call(causal=1, Sq=400, Sk=300) == -2


def test_bwd_onepass_fails_closed(h):
    lib = h.lib
    need = h.bwd_onepass_workspace_size(1, 2, 128)
    assert need >= 2 * 128 * 128 * 4 + 2 * 128 * 4                 # dQ accumulator and Delta at least

    def call(ws=A, wsb=need, causal=0, Sq=128, Sk=128, D=128, dq=A):
        return lib.attn_bwd_onepass(A, A, A, A, A, A, dq, A, A, 1, 2, 2, Sq, Sk, D, 0.088, causal, ws, wsb, None)

    assert call(wsb=need - 1) == -4
    assert call(ws=None) == -1
    assert call(dq=None) == -1
    assert call(dq=MIS) == -3
    assert call(D=96) == -2
    assert call(causal=1, Sq=256, Sk=128) == -2
    # a counter that is not 4-byte aligned is refused before anything is launched
    assert lib.attn_selftest_counter_wait(ctypes.c_void_p(0x20001), None, 1000) == -3


def test_error_strings(h):
    for c in (0, -1, -2, -3, -4, -5, -6, -99):
        assert isinstance(h.lib.attn_error_string(c), bytes)


def test_binding_refuses_fp32_inputs(h):
    import torch

    with pytest.raises((TypeError, ValueError)):
        h.attn_fwd(torch.zeros(1, 1, 8, 128), torch.zeros(1, 1, 8, 128), torch.zeros(1, 1, 8, 128))
