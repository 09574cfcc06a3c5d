"""The library's once-per-device set-up table (kernel shared-memory opt-ins
and the static scratch's address are per device): built from its header with
the host C++ compiler and exercised with racing threads, several device
ordinals, a failing set-up and out-of-range ordinals.  No GPU needed."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_per_device_table(tmp_path):
    exe = tmp_path / "per_device_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread",
                    "-I", os.path.join(ROOT, "include"),
                    "-I", os.path.join(ROOT, "block_sparse_local_raster_b200", "csrc"),
                    os.path.join(ROOT, "tests", "cpp", "per_device_check.cpp"),
                    "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip() == "ok", r.stdout + r.stderr
