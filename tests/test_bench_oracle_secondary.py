"""bench.py's oracle timings beside the secondary rows run on the CPU and
report positive rates for quantize, dequantize and the decode-shaped forward."""

import math

import bench


def test_oracle_secondary_small_sample():
    res = bench.oracle_secondary("cpu", row_div=256)
    for key, field in (("quantize", "GB/s"), ("dequant_bf16", "GB/s"), ("gemv_gate_14336x4096_M16", "us_per_call")):
        v = res[key][field]
        assert v > 0 and math.isfinite(v), key
    assert "1/256" in res["sample"]


def test_cpu_model_is_named():
    assert isinstance(bench.cpu_model(), str) and bench.cpu_model()
    assert bench.cores_used() >= 1
