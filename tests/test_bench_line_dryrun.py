"""Dry run of bench.py's default arm on the CPU: the JSON line it prints.

Every GPU-touching piece (the layer step, the timed loop, the library's
timing records, the clock sampler and the secondary measurements) is a fake
returning fixed numbers, so the test checks the line's assembly: every key
of the measurement contract is present with the right type, the roofline and
whole-job figures follow from the fakes' numbers, the default run carries the
32-layer stack row, and the flags add or drop their fields without changing
the rest.
"""

import argparse
import json

import pytest
import torch

import bench
from bit_nf4_quantized_blk_b200 import binding

STEP_MS = 8.0
GEMM_MS_PER_STEP = 6.0


class FakeStep:
    def __init__(self, device, M=bench.M_TOKENS):
        self.runs = 0
        self.two_stream_runs = 0

    def run(self):
        self.runs += 1

    def run_two_streams(self):
        self.two_stream_runs += 1

    def check_status(self):
        pass

    def host_buffers(self):
        return 2_217_213_952, 1_347_420_160

    def e2e_timed(self, steps, warmup, world):
        return 45.0


class FakeClock:
    def __init__(self, idx):
        pass

    def start(self):
        pass

    def stop(self, window):
        return {"sm_mhz": 1650.0, "sm_max_mhz": 1965.0, "reasons": ["sw_power_cap"], "samples": 10}

    @staticmethod
    def around(device_index, fn):
        return fn(), {"sm_mhz": 1900.0, "sm_max_mhz": 1965.0, "reasons": [], "samples": 4}


@pytest.fixture
def dry(monkeypatch):
    made = {}

    def fake_step(device, M=bench.M_TOKENS):
        made["step"] = FakeStep(device, M)
        return made["step"]

    steps_recorded = {}

    def timed(fn, steps, warmup, world, window=None):
        for _ in range(warmup + steps):
            fn()
        steps_recorded["n"] = steps + warmup
        if window is not None:
            window[:] = [0.0, 1.0]
        return STEP_MS

    def timing_read(family):
        n = steps_recorded.get("n", 1)
        return {"gemm": (GEMM_MS_PER_STEP * n, 14 * n)}.get(family, (0.5 * n, 10 * n))

    from bit_nf4_quantized_blk_b200 import build

    monkeypatch.setattr(build, "build", lambda *a, **k: None)
    monkeypatch.setattr(bench, "LayerStep", fake_step)
    monkeypatch.setattr(bench, "ClockSampler", FakeClock)
    monkeypatch.setattr(bench, "timed", timed)
    monkeypatch.setattr(torch.cuda, "synchronize", lambda *a, **k: None)
    monkeypatch.setattr(binding, "qlora_timing_enable", lambda on: None)
    monkeypatch.setattr(binding, "qlora_timing_read", timing_read)
    monkeypatch.setattr(torch.cuda, "empty_cache", lambda: None)
    monkeypatch.setattr(bench, "bench_quantize_dequant", lambda clock=None: {
        "quantize": {"ms": 1.0, "GB/s": 5000.0}, "dequant_bf16": {"ms": 1.0, "GB/s": 6000.0}})
    monkeypatch.setattr(bench, "bench_gemv", lambda: {"M=1": {"us": 25.0, "GB/s": 1200.0,
                                                             "write_flush": {"us": 30.0, "GB/s": 1000.0}},
                                                     "method": "rotation"})
    monkeypatch.setattr(bench, "bench_merge", lambda: {"ms": 0.2, "GB/s": 2700.0})
    monkeypatch.setattr(bench, "bench_stack", lambda: {"quantize": {"ms": 6.0, "GB/s": 5200.0},
                                                      "fwd_bwd": {"ms": 250.0, "TFLOP/s": 920.0}})
    monkeypatch.setattr(bench, "cpu_cases", lambda device, tokens: [])
    monkeypatch.setattr(bench, "oracle_sample_step", lambda cases, row_div, tokens: (0.1, 72.0))
    monkeypatch.setattr(bench, "oracle_secondary", lambda device: {"quantize": {"GB/s": 0.04}})
    return made


def _args(**kw):
    base = dict(gpus=1, steps=5, warmup=3, impl="ours", no_extras=False, no_cpu=False, streams=1, no_stack=False)
    base.update(kw)
    return argparse.Namespace(**base)


def _line(capsys, args):
    bench.run_ours(args, 0, 1, 0)
    out = capsys.readouterr().out.strip().splitlines()
    assert len(out) == 1, out
    return json.loads(out[0])


def test_default_line_has_every_contract_key(dry, capsys):
    d = _line(capsys, _args())
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "cpu_baseline", "e2e",
                "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["higher_is_better"] is True and d["scaling"] == "weak" and d["vs_baseline"] is None
    assert d["value"] == pytest.approx(bench.step_flops() / (STEP_MS / 1e3) / 1e12)
    assert "workload" in d["config"] and "streams" not in d["config"]
    r = d["roofline"]
    for key in ("bound", "achieved", "peak", "unit", "frac", "traffic"):
        assert key in r, key
    assert r["bound"] == "tensor" and r["unit"] == "TFLOP/s"
    assert r["achieved"] == pytest.approx(bench.gemm_flops_per_step() / (GEMM_MS_PER_STEP / 1e3) / 1e12)
    assert r["frac"] == pytest.approx(r["achieved"] / r["peak"])
    assert r["peak"] == bench.load_peaks()[0].get("bf16_tflops", bench.FALLBACK_PEAKS["bf16_tflops"])  # burst
    assert r["frac_clock_normalized"] == pytest.approx(r["achieved"] / (r["peak"] * 1650.0 / r["peak_clock_mhz"]))
    cb = d["cpu_baseline"]
    for key in ("value", "unit", "cores", "kind", "sample", "cpu_model", "nproc", "secondary"):
        assert key in cb, key
    assert cb["kind"] == "oracle"
    e = d["e2e"]
    for key in ("value", "unit", "h2d_bytes_per_step", "d2h_bytes_per_step"):
        assert key in e, key
    assert e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == (14 + 4 * 10) * 5
    st = d["secondary"]["stack_32x7_8192tok"]  # config 5 is part of the default run
    assert "frac_hbm" in st["quantize"] and "frac_bf16_burst" in st["fwd_bwd"] and st["clocks"]["samples"] == 4
    g = d["secondary"]["gemv_gate_14336x4096"]["M=1"]
    assert "frac_hbm" in g and "frac_hbm" in g["write_flush"]
    assert dry["step"].runs == 1 + 3 + 5 and dry["step"].two_stream_runs == 0


def test_flags(dry, capsys):
    d = _line(capsys, _args(streams=2, no_stack=True, no_cpu=True, no_extras=True))
    assert d["config"]["streams"].startswith("projections alternate")
    assert "stack_32x7_8192tok" not in d.get("secondary", {})
    assert "cpu_baseline" not in d
    assert dry["step"].two_stream_runs == 3 + 5 and dry["step"].runs == 1


def test_gemm_traffic_follows_the_source_digest(monkeypatch, tmp_path):
    """roofline.traffic comes from the committed capture only while the GEMM's
    sources hash to the digest recorded beside it; otherwise it is null."""
    import hashlib
    import os

    h = hashlib.sha256()
    for rel in bench.GEMM_SOURCES:
        with open(os.path.join(bench.ROOT, "bit_nf4_quantized_blk_b200", rel), "rb") as f:
            h.update(f.read())
    current = tmp_path / "current.md"
    current.write_text(f"traffic_bytes_per_launch: 123\nsource_digest: {h.hexdigest()[:16]}\n")
    monkeypatch.setattr(bench, "GEMM_TRAFFIC_PROFILE", str(current))
    assert bench.gemm_traffic_per_launch() == 123
    stale = tmp_path / "summary.md"
    stale.write_text("traffic_bytes_per_launch: 123\nsource_digest: 0000000000000000\n")
    monkeypatch.setattr(bench, "GEMM_TRAFFIC_PROFILE", str(stale))
    assert bench.gemm_traffic_per_launch() is None
    monkeypatch.setattr(bench, "GEMM_TRAFFIC_PROFILE", str(tmp_path / "missing.md"))
    assert bench.gemm_traffic_per_launch() is None
