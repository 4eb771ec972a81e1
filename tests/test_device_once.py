"""Host-side helpers of the launchers: per-device one-time kernel setup.

The dynamic shared-memory limit of a kernel is a property of one device's
context, so the library's launchers remember per device ordinal whether they
have set it (device_once.h).  These checks build a small C++ program against
that header with the host compiler; no GPU is involved.
"""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
CSRC = os.path.join(ROOT, "bit_nf4_quantized_blk_b200", "csrc")
SRC = os.path.join(ROOT, "tests", "native", "device_once_test.cc")


@pytest.mark.skipif(shutil.which("g++") is None, reason="needs the host C++ compiler")
def test_device_once_helpers():
    out_dir = os.path.join(ROOT, "_build", "tests")
    os.makedirs(out_dir, exist_ok=True)
    exe = os.path.join(out_dir, "device_once_test")
    subprocess.run(["g++", "-std=c++17", "-O1", "-Wall", "-Werror", "-pthread", "-I", CSRC, SRC, "-o", exe],
                   check=True, capture_output=True, text=True)
    res = subprocess.run([exe], capture_output=True, text=True, timeout=60)
    assert res.returncode == 0 and res.stdout.strip() == "ok", res.stdout + res.stderr


def test_every_launcher_uses_per_device_setup():
    """No launcher keeps a process-wide 'already configured' flag."""
    offenders = []
    for name in sorted(os.listdir(CSRC)):
        if not name.endswith((".cu", ".cuh")):
            continue
        with open(os.path.join(CSRC, name)) as f:
            for no, line in enumerate(f, 1):
                if "cudaFuncSetAttribute" in line:
                    continue
                if "static bool configured" in line or "static int cached" in line:
                    offenders.append(f"{name}:{no}")
    assert not offenders, offenders
