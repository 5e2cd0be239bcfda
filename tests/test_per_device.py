"""The per-device bookkeeping of the kernels' one-time launch attributes (CPU only).

Launch attributes such as the maximum dynamic shared memory are recorded per
device, so the library sets them once on every device it launches on.  This
compiles a host-only C++ check of that bookkeeping (csrc/per_device.h) with g++
and runs it: once per device, retried after a failure, untracked devices set
every time, and many threads racing on the first call."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_per_device_once(tmp_path):
    exe = tmp_path / "per_device_check"
    src = os.path.join(ROOT, "tests", "per_device_check.cpp")
    inc = os.path.join(ROOT, "qk_normed_latent_qkn_b200", "csrc")
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-I", inc, src, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
