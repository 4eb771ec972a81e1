"""The debug library (QLORA_CHECKS: index and alignment tests compiled into
the kernels, a failed test recording QLORA_ERR_CHECK and skipping the access)
runs small odd-shaped calls through every entry point with no failed test and
gives the same bits as the default library.

Each library runs in its own child process (tests/checks_cases.py), so the two
builds never share a process."""

import os
import subprocess
import sys

import pytest
import torch

from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _run(lib: str, out: str) -> dict:
    proc = subprocess.run([sys.executable, os.path.join(HERE, "checks_cases.py"), lib, out], capture_output=True,
                          text=True, timeout=600)
    assert proc.returncode == 0, proc.stdout[-2000:] + proc.stderr[-2000:]
    return torch.load(out)


def test_checks_build_matches_default_build(tmp_path):
    from bit_nf4_quantized_blk_b200 import build

    default_lib = build.build()
    checks_lib = build.build(checks=True)
    ref = _run(default_lib, str(tmp_path / "default.pt"))
    chk = _run(checks_lib, str(tmp_path / "checks.pt"))
    assert sorted(ref) == sorted(chk)
    # The checks are live in the debug library's device code, compiled away in the default one.
    assert int(ref.pop("checks_probe")) == 0
    assert int(chk.pop("checks_probe")) == 8  # QLORA_ERR_CHECK
    for key in ref:
        if key.endswith("/status"):
            assert int(chk[key]) == 0, f"{key}: status {int(chk[key])} under the checks build"
            assert int(ref[key]) == 0, key
        else:
            assert torch.equal(ref[key], chk[key]), key
