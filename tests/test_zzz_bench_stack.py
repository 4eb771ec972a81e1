"""GPU: bench.py's opt-in stack measurement runs end to end (4 of the 32 layers).

bench_stack asserts that the quantize status and the linear workspace status
are clean; the chain's wiring is checked on the CPU (test_bench_stack_dryrun)
and its numerics by the 32-layer parity test (test_gpu_stack).
"""

import math

import pytest

import bench
from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


def test_bench_stack_runs():
    require_gpu()
    res = bench.bench_stack(steps=1, warmup=0, layers=4)
    assert res["quantize"]["weights"] == 4 * sum(p.n * p.k for p in bench.workloads.LAYER7B)
    for phase, key in (("quantize", "GB/s"), ("fwd_bwd", "TFLOP/s")):
        assert res[phase]["ms"] > 0 and math.isfinite(res[phase][key]), phase
