"""Host-side logic of the scoped device switch every entry point uses: the
library launches on the state buffer's device and must hand the caller's
current device back on every return path.  Compiled with g++ against a fake
device API, so it runs without a GPU."""

import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "delta_rule_recurrent_scan_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "native", "device_guard_check.cpp")


@pytest.mark.skipif(shutil.which("g++") is None, reason="g++ not available")
def test_scoped_device_restores_the_callers_device(tmp_path):
    exe = tmp_path / "device_guard_check"
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-I", CSRC, SRC, "-o", str(exe)], check=True)
    r = subprocess.run([str(exe)], capture_output=True, text=True)
    assert r.returncode == 0, r.stdout + r.stderr
    assert r.stdout.strip() == "ok"
