"""The stored dS^T tile layout of attn_bwd_dsbuf (csrc/ds_layout.h) on the
CPU: a bijection of the tile, 512 contiguous bytes per warp store, and the
core-block strides the dQ product's operand descriptor assumes.  Compiled
with g++."""
import os
import subprocess
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_ds_tile_layout():
    src = os.path.join(ROOT, "tests", "ds_layout_check.cc")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "ds_layout_check")
        subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-o", exe, src], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "ds_layout ok" in r.stdout
