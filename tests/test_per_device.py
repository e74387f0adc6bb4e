"""The per-device one-time kernel setup (csrc/per_device.h) on the CPU: each
device ordinal runs its setup once, independently of the others; a failed
setup is retried; concurrent first calls run it once.  A process driving two
real GPUs cannot be exercised here (every GPU run has one device), so the
logic is checked with ordinals alone, compiled with g++."""
import os
import subprocess
import tempfile

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_per_device_once():
    src = os.path.join(ROOT, "tests", "per_device_check.cc")
    with tempfile.TemporaryDirectory() as tmp:
        exe = os.path.join(tmp, "per_device_check")
        subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-Wall", "-o", exe, src], check=True)
        r = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stderr
    assert "per_device ok" in r.stdout
