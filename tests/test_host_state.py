"""Host-side state of the library, tested without a GPU: the per-device
memo behind the GEMM kernels' shared-memory attribute and the quantize
kernels' occupancy (fp8_math_b200/csrc/devcache.h) is compiled with the host
C++ compiler into a small test program, which checks that each (kernel,
device) pair is set up once, that values stay per device, that failures are
retried, and that concurrent first calls from 16 threads agree."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="no host C++ compiler")
def test_per_device_memo(tmp_path):
    exe = tmp_path / "devcache_test"
    subprocess.check_call(["g++", "-std=c++17", "-O1", "-pthread", "-I", os.path.join(ROOT, "fp8_math_b200", "csrc"),
                           os.path.join(ROOT, "tests", "host", "devcache_test.cpp"), "-o", str(exe)])
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
