"""The host-side per-device memos of the library (csrc/per_device.h), compiled on their own
with the host compiler and run with several threads and device ids: a kernel attribute is
set once per device (a failure is retried, other devices are unaffected) and device
properties are cached per device."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs a host C++ compiler")
def test_per_device_memos(tmp_path):
    exe = tmp_path / "per_device_test"
    subprocess.run(["g++", "-std=c++17", "-O1", "-pthread", "-Wall", "-Werror",
                    "-I", os.path.join(ROOT, "int8_mixed_precision_vectorwise_b200", "csrc"),
                    os.path.join(ROOT, "tests", "cpp", "per_device_test.cpp"), "-o", str(exe)],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True, timeout=60)
    assert r.returncode == 0 and r.stdout.strip().endswith("ok"), r.stdout + r.stderr
