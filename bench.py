"""Benchmark of the QLoRA NF4 linear hot path on B200 (one JSON line on rank 0).

Step (the headline workload): one training-shaped 7B decoder layer's seven
projections (q 4096x4096, k/v 1024x4096, o 4096x4096, gate/up 14336x4096,
down 4096x14336) at 8192 tokens, LoRA r = 16, alpha = 32:
  quantize + double-quantize all seven fp32 weights (one batched call),
  forward of every projection, backward (dX, dA, dB) of every projection.
Metric: algorithmic TFLOP/s of the forward + backward,
  4 M sum(N K) + 6 M r sum(N + K) = 7.211 TFLOP per step per GPU
(the quantize work is inside the timed step but not counted as FLOPs).

Multi-GPU: one process per GPU (torchrun), each rank runs the same step on
its own replica (the method has no exchange step on this path), so scaling is
weak; time is the max over ranks of CUDA-event time.

Also reported on rank 0 (not the headline): quantize and dequantize GB/s over
the 168 OPT-1.3B-shaped tensors, dequant-GEMV GB/s on the 14336 x 4096 gate
projection at M = 1, 4, 16 (L2 flushed before every call), the end-to-end
number with pinned host buffers, and the CPU oracle baseline.
"""

from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np
import torch
import torch.distributed as dist

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from bit_nf4_quantized_blk_b200 import binding, workloads  # noqa: E402

R = 16
ALPHA = 32.0
M_TOKENS = 8192
METRIC = "QLoRA linear fwd+bwd TFLOP/s @8192 tok; dequant-GEMV & quantize GB/s vs HBM"
WORKLOAD = ("7B decoder layer, 7 NF4+DQ projections (q 4096x4096, k/v 1024x4096, o 4096x4096, "
            "gate/up 14336x4096, down 4096x14336), 8192 tokens, r=16 alpha=32: "
            "quantize+DQ, forward, backward (dX, dA, dB)")
PEAKS_PATH = os.path.join(ROOT, "MEASURED_PEAKS.json")
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def step_flops(M=M_TOKENS, r=R):
    snk = sum(p.n * p.k for p in workloads.LAYER7B)
    snpk = sum(p.n + p.k for p in workloads.LAYER7B)
    return 4 * M * snk + 6 * M * r * snpk


def gemm_flops_per_step(M=M_TOKENS, r=R):
    # forward GEMM: 2 M N (K + r); backward-input GEMM: 2 M K (N + r)
    return sum(2 * M * p.n * (p.k + r) + 2 * M * p.k * (p.n + r) for p in workloads.LAYER7B)


def load_peaks():
    if os.path.exists(PEAKS_PATH):
        with open(PEAKS_PATH) as f:
            return json.load(f), "measured"
    return FALLBACK_PEAKS, "fallback"


# ---------------------------------------------------------------------------
# Clock sampling during the timed region
# ---------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi clock / throttle-reason samples every 50 ms; `stop(window)`
    keeps those stamped inside the host wall-clock window of the timed region
    (all samples under load if none fall inside it)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device_index: int):
        self.device_index = device_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.device_index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
            time.sleep(0.5)  # let the first samples arrive before the load starts
        except (OSError, FileNotFoundError):
            self.proc = None

    @staticmethod
    def _stamp(text):
        try:
            return datetime.datetime.strptime(text.strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
        except ValueError:
            return None

    @staticmethod
    def around(device_index, fn):
        """(fn(), clocks sampled while it ran); clocks is None when
        `device_index` is None or nvidia-smi is unavailable."""
        if device_index is None:
            return fn(), None
        c = ClockSampler(device_index)
        c.start()
        t0 = time.time()
        out = fn()
        t1 = time.time()
        return out, c.stop([t0, t1])

    def stop(self, window=None):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) < 10:
                    continue
                try:
                    rows.append((self._stamp(parts[0]), float(parts[2]), float(parts[3]), parts[6:10]))
                except ValueError:
                    continue
        os.unlink(self.path)
        inside = rows
        scope = "all samples"
        if window is not None:
            sel = [r for r in rows if r[0] is not None and window[0] <= r[0] <= window[1]]
            if sel:
                inside, scope = sel, "timed region"
        if not inside:
            return None
        reasons = set()
        for r in inside:
            for name, val in zip(names, r[3]):
                if val.lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r[1] for r in inside), "sm_max_mhz": max(r[2] for r in inside),
                "reasons": sorted(reasons), "samples": len(inside), "scope": scope, "interval_ms": 50}


# ---------------------------------------------------------------------------
# The layer step
# ---------------------------------------------------------------------------

class LayerStep:
    """Resident inputs, outputs and workspaces of one 7B layer step."""

    def __init__(self, device, M=M_TOKENS):
        self.M = M
        self.cases = [workloads.layer7b_case(t, m=M, device=device) for t in range(7)]
        self.outs = [binding.NF4Weight.empty(c.proj.n, c.proj.k, device=device) for c in self.cases]
        self.qws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(self.outs), dtype=torch.uint8, device=device)
        self.dstat = torch.zeros(1, dtype=torch.int32, device=device)
        lws = max(binding.qlora_linear_ws_bytes(M, c.proj.n, c.proj.k, c.r) for c in self.cases)
        self.lws = torch.empty(lws, dtype=torch.uint8, device=device)
        binding.qlora_workspace_reset(self.lws)
        self.Y = [torch.empty((M, c.proj.n), dtype=torch.bfloat16, device=device) for c in self.cases]
        self.dX = [torch.empty((M, c.proj.k), dtype=torch.bfloat16, device=device) for c in self.cases]
        self.dA = [torch.empty((c.r, c.proj.k), dtype=torch.float32, device=device) for c in self.cases]
        self.dB = [torch.empty((c.proj.n, c.r), dtype=torch.float32, device=device) for c in self.cases]
        self.U = [torch.empty((M, c.r), dtype=torch.float32, device=device) for c in self.cases]

    def run(self):
        binding.qlora_nf4_quantize_batched([c.W for c in self.cases], self.outs, self.qws, d_status=self.dstat)
        for c, o, Y, U in zip(self.cases, self.outs, self.Y, self.U):
            binding.qlora_linear_fwd(o, c.X, c.A, c.B, c.r, c.s, Y, U, self.lws)
        for c, o, dX, dA, dB, U in reversed(list(zip(self.cases, self.outs, self.dX, self.dA, self.dB, self.U))):
            binding.qlora_linear_bwd(o, c.X, c.dY, c.A, c.B, c.r, c.s, dX, 0, dA, dB, self.lws, U=U)

    def run_two_streams(self):
        """run() with the projections' calls alternating over two streams, one
        workspace per stream, so that one projection's HBM-bound kernels can
        run beside another's GEMM.  A backward waits for its own forward (its
        saved U); the step ends when both streams have finished.  The outputs
        are bit-identical to run()'s."""
        if getattr(self, "_streams", None) is None:
            self._ws2 = torch.empty_like(self.lws)
            binding.qlora_workspace_reset(self._ws2)
            self._streams = [torch.cuda.Stream(), torch.cuda.Stream()]
        main = torch.cuda.current_stream()
        wss, streams = [self.lws, self._ws2], self._streams
        binding.qlora_nf4_quantize_batched([c.W for c in self.cases], self.outs, self.qws, d_status=self.dstat)
        for st in streams:
            st.wait_stream(main)
        fwd_done = []
        for i, (c, o, Y, U) in enumerate(zip(self.cases, self.outs, self.Y, self.U)):
            with torch.cuda.stream(streams[i % 2]):
                binding.qlora_linear_fwd(o, c.X, c.A, c.B, c.r, c.s, Y, U, wss[i % 2])
                ev = torch.cuda.Event()
                ev.record(streams[i % 2])
                fwd_done.append(ev)
        for j, i in enumerate(reversed(range(len(self.cases)))):
            c, o = self.cases[i], self.outs[i]
            with torch.cuda.stream(streams[j % 2]):
                streams[j % 2].wait_event(fwd_done[i])
                binding.qlora_linear_bwd(o, c.X, c.dY, c.A, c.B, c.r, c.s, self.dX[i], 0, self.dA[i], self.dB[i],
                                         wss[j % 2], U=self.U[i])
        for st in streams:
            main.wait_stream(st)

    def check_status(self):
        assert self.dstat.item() == 0, "quantize reported non-finite input"
        for ws in (self.lws, getattr(self, "_ws2", None)):
            if ws is not None:
                st = binding.qlora_workspace_status(ws)
                assert st == 0, f"device status {st}"

    # end-to-end: host buffers in, host buffers out
    def host_buffers(self):
        pin = lambda t: t.cpu().pin_memory()  # noqa: E731
        self.h_in = [(pin(c.W), pin(c.X), pin(c.dY), pin(c.A), pin(c.B)) for c in self.cases]
        self.h_out = [(torch.empty(y.shape, dtype=y.dtype).pin_memory(), torch.empty(dx.shape, dtype=dx.dtype).pin_memory(),
                       torch.empty(da.shape, dtype=da.dtype).pin_memory(), torch.empty(db.shape, dtype=db.dtype).pin_memory())
                      for y, dx, da, db in zip(self.Y, self.dX, self.dA, self.dB)]
        h2d = sum(sum(t.numel() * t.element_size() for t in grp) for grp in self.h_in)
        d2h = sum(sum(t.numel() * t.element_size() for t in grp) for grp in self.h_out)
        return h2d, d2h

    def run_set(self, k):
        """One step on device buffer set k (inputs, outputs; the quantized state,
        U and the workspace are shared: the compute stream runs steps in order)."""
        ins, outs = self.sets_in[k], self.sets_out[k]
        binding.qlora_nf4_quantize_batched([i[0] for i in ins], self.outs, self.qws, d_status=self.dstat)
        for c, o, (W, X, dY, A, B), (Y, dX, dA, dB), U in zip(self.cases, self.outs, ins, outs, self.U):
            binding.qlora_linear_fwd(o, X, A, B, c.r, c.s, Y, U, self.lws)
        for c, o, (W, X, dY, A, B), (Y, dX, dA, dB), U in reversed(list(zip(self.cases, self.outs, ins, outs, self.U))):
            binding.qlora_linear_bwd(o, X, dY, A, B, c.r, c.s, dX, 0, dA, dB, self.lws, U=U)

    def e2e_timed(self, steps, warmup, world):
        """End to end, milliseconds per step: every step uploads its inputs
        (fp32 weights, X, dY, A, B) from pinned host memory, runs the layer step
        and downloads its outputs (Y, dX, dA, dB), pipelined as an input
        pipeline would be: step i + 1's upload and step i - 1's download run on
        their own streams while step i computes, with two device buffer sets
        (a set is refilled only after the compute that read it, and rewritten
        only after its outputs were downloaded)."""
        mk = lambda t: torch.empty_like(t)  # noqa: E731
        self.sets_in = [[(c.W, c.X, c.dY, c.A, c.B) for c in self.cases],
                        [(mk(c.W), mk(c.X), mk(c.dY), mk(c.A), mk(c.B)) for c in self.cases]]
        self.sets_out = [list(zip(self.Y, self.dX, self.dA, self.dB)),
                         [(mk(y), mk(dx), mk(da), mk(db)) for y, dx, da, db in zip(self.Y, self.dX, self.dA, self.dB)]]
        for (W, X, dY, A, B), c in zip(self.sets_in[1], self.cases):  # same inputs in both sets
            for dst, src in zip((W, X, dY, A, B), (c.W, c.X, c.dY, c.A, c.B)):
                dst.copy_(src)
        s_h, s_c, s_d = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
        ev_in = [torch.cuda.Event(), torch.cuda.Event()]
        ev_done = [torch.cuda.Event(), torch.cuda.Event()]
        ev_out = [torch.cuda.Event(), torch.cuda.Event()]
        h_in = [t for grp in self.h_in for t in grp]
        h_out = [t for grp in self.h_out for t in grp]

        def step(i):
            k = i % 2
            with torch.cuda.stream(s_h):
                if i >= 2:
                    s_h.wait_event(ev_done[k])
                for dev, host in zip([t for grp in self.sets_in[k] for t in grp], h_in):
                    dev.copy_(host, non_blocking=True)
                ev_in[k].record(s_h)
            with torch.cuda.stream(s_c):
                s_c.wait_event(ev_in[k])
                if i >= 2:
                    s_c.wait_event(ev_out[k])
                self.run_set(k)
                ev_done[k].record(s_c)
            with torch.cuda.stream(s_d):
                s_d.wait_event(ev_done[k])
                for host, dev in zip(h_out, [t for grp in self.sets_out[k] for t in grp]):
                    host.copy_(dev, non_blocking=True)
                ev_out[k].record(s_d)

        for i in range(warmup):
            step(i)
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        start.record(s_h)
        s_c.wait_event(start)
        s_d.wait_event(start)
        for i in range(warmup, warmup + steps):
            step(i)
        stop.record(s_d)  # the last download follows the last compute, which follows every upload
        torch.cuda.synchronize()
        if world > 1:
            dist.barrier()
        ms = start.elapsed_time(stop) / steps
        if world > 1:
            ms = max_over_ranks(ms, "cuda")
        self.sets_in = self.sets_out = None
        return ms


def max_over_ranks(value: float, device) -> float:
    """The largest `value` over all ranks (every rank gets the same answer)."""
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(units_per_rank: float, world: int, ms: float) -> float:
    """Whole-job throughput: the units all ranks processed / the slowest rank's time."""
    return units_per_rank * world / (ms / 1e3)


def timed(fn, steps, warmup, world, window=None):
    """Device time per step of `steps` calls after `warmup` untimed ones,
    bracketed by a barrier and a synchronize; the max over ranks.  `window`
    (a list) receives the host wall-clock span of the timed calls."""
    for _ in range(warmup):
        fn()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start, stop = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    t0 = time.time()
    start.record()
    for _ in range(steps):
        fn()
    stop.record()
    torch.cuda.synchronize()
    t1 = time.time()
    if window is not None:
        window[:] = [t0, t1]
    if world > 1:
        dist.barrier()
    ms = start.elapsed_time(stop) / steps
    if world > 1:
        ms = max_over_ranks(ms, "cuda")
    return ms


# ---------------------------------------------------------------------------
# Secondary measurements (rank 0): quantize / dequant / GEMV / merge rows
# ---------------------------------------------------------------------------

def timed_reps(fn, reps, warmup, before=None):
    """Per-call device times (ms) of `reps` calls after `warmup` untimed ones,
    every call bracketed by its own pair of events on the current stream;
    `before` (untimed) runs ahead of each call.  A device-side sleep queued
    first keeps the GPU busy while the host enqueues every timed call, so the
    calls run back to back and no interval holds time the device spent
    waiting for the host to launch the call's kernels."""
    for _ in range(warmup):
        if before is not None:
            before(0)
        fn()
    torch.cuda.synchronize()
    t0 = time.perf_counter()
    if before is not None:
        before(0)
    fn()
    host_s = time.perf_counter() - t0  # host time to enqueue one call
    torch.cuda.synchronize()
    torch.cuda._sleep(int(min(2.0, 2.0 * reps * host_s + 1e-3) * 2.0e9))  # cycles at about 2 GHz
    evs = []
    for i in range(reps):
        if before is not None:
            before(i)
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        evs.append((a, b))
    torch.cuda.synchronize()
    return [a.elapsed_time(b) for a, b in evs]


def rep_stats(ms_list):
    return {"ms": statistics.median(ms_list), "ms_min": min(ms_list), "reps": len(ms_list)}

def l2_flush_buffer():
    size = 2 * torch.cuda.get_device_properties(0).L2_cache_size
    return torch.empty(max(size, 256 << 20) // 4, dtype=torch.float32, device="cuda")


def bench_quantize_dequant(reps=20, clock=None):
    """Config 2: quantize + DQ, then bf16 dequantize, of the 168 OPT-1.3B-shaped
    tensors (one batched call each), `reps` timed calls of each (median and
    minimum), with the SM clocks sampled over each row's calls."""
    items = workloads.opt13b_weight_shapes()
    Ws = [workloads.opt13b_weight(layer, t, device="cuda") for layer, t, _ in items]
    outs = [binding.NF4Weight.empty(p.n, p.k) for _, _, p in items]
    ws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
    dstat = torch.zeros(1, dtype=torch.int32, device="cuda")
    n = sum(p.n * p.k for _, _, p in items)
    res = {}
    q_clock = ClockSampler.around(clock, lambda: timed_reps(
        lambda: binding.qlora_nf4_quantize_batched(Ws, outs, ws, d_status=dstat), reps, 3))
    assert dstat.item() == 0
    ys = [torch.empty((p.n, p.k), dtype=torch.bfloat16, device="cuda") for _, _, p in items]
    d_clock = ClockSampler.around(clock, lambda: timed_reps(
        lambda: binding.qlora_nf4_dequantize_batched(outs, ys, 0), reps, 3))
    q_bytes = n * (4 + 0.5 + 1 / 64) + 4 * sum(o.c2.numel() + 1 for o in outs)
    d_bytes = n * (0.5 + 1 / 64 + 2) + 4 * sum(o.c2.numel() + 1 for o in outs)
    del Ws, ys
    for name, (ms_list, clocks), nbytes, bpw in (("quantize", q_clock, q_bytes, 4.5159),
                                                   ("dequant_bf16", d_clock, d_bytes, 2.5159)):
        st = rep_stats(ms_list)
        res[name] = {"weights": n, **st, "GB/s": nbytes / st["ms"] / 1e6, "GB/s_best": nbytes / st["ms_min"] / 1e6,
                     "bytes_per_weight": bpw, "clocks": clocks}
    return res


def bench_gemv(reps=100, copies=8):
    """Config 3: the decode-shaped forward on the 14336 x 4096 gate at M = 1,
    4, 16.  `copies` quantized copies of the gate (8 x 31 MB, more than the
    L2) are used in turn, so every call reads its weight from HBM with no
    flush kernel in between; the old figure with a 2 x L2 write flush before
    every call (whose dirty lines the GEMV then has to write back) is kept
    beside it for comparison."""
    case = workloads.gemv_case(16, device="cuda")
    qws = torch.empty(binding.qlora_nf4_sizes(14336, 4096)["ws_bytes"], dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(copies):
        o = binding.NF4Weight.empty(14336, 4096)
        binding.qlora_nf4_quantize(case.W, o, qws)
        outs.append(o)
    flush = l2_flush_buffer()
    res = {}
    for M in (1, 4, 16):
        X = workloads.normal_bf16((M, 4096), 1.0, 3000 + M, device="cuda")
        Y = torch.empty((M, 14336), dtype=torch.bfloat16, device="cuda")
        ws = torch.empty(binding.qlora_linear_ws_bytes(M, 14336, 4096, 16), dtype=torch.uint8, device="cuda")
        binding.qlora_workspace_reset(ws)
        cur = [0]

        def fwd():
            binding.qlora_linear_fwd(outs[cur[0] % copies], X, case.A, case.B, 16, case.s, Y, None, ws)
            cur[0] += 1

        rot = rep_stats(timed_reps(fwd, reps, 3))
        cur[0] = 0
        fl = rep_stats(timed_reps(lambda: binding.qlora_linear_fwd(outs[0], X, case.A, case.B, 16, case.s, Y, None, ws),
                                  reps // 2, 3, before=lambda i: flush.zero_()))
        o = outs[0]
        nbytes = (o.packed.numel() + o.qscale.numel() + 4 * o.c2.numel() + 4 + 2 * (case.A.numel() + case.B.numel())
                  + 2 * M * (4096 + 14336))
        res[f"M={M}"] = {"us": rot["ms"] * 1e3, "us_min": rot["ms_min"] * 1e3, "GB/s": nbytes / rot["ms"] / 1e6,
                         "bytes": nbytes, "reps": rot["reps"],
                         "write_flush": {"us": fl["ms"] * 1e3, "GB/s": nbytes / fl["ms"] / 1e6}}
        assert binding.qlora_workspace_status(ws) == 0
    res["method"] = (f"{copies} quantized copies of the gate used in turn (no flush kernel); write_flush: a 2 x L2 "
                     "write before every call")
    return res


def bench_merge(reps=10):
    """Merged bf16 weights W_hat + s B A of the 7B layer's seven projections
    (r = 16): one qlora_merge per projection, the seven timed together."""
    cases = [workloads.linear_case(p, 1, 16, 32.0, 4, 0, t, "cuda", with_dy=False)
             for t, p in enumerate(workloads.LAYER7B)]
    outs = [binding.NF4Weight.empty(c.proj.n, c.proj.k) for c in cases]
    ws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
    dstat = torch.zeros(1, dtype=torch.int32, device="cuda")
    binding.qlora_nf4_quantize_batched([c.W for c in cases], outs, ws, d_status=dstat)
    for c in cases:
        c.W = None
    ys = [torch.empty((c.proj.n, c.proj.k), dtype=torch.bfloat16, device="cuda") for c in cases]

    def run():
        for c, o, y in zip(cases, outs, ys):
            binding.qlora_merge(o, c.A, c.B, c.r, c.s, y, 0)

    ms = timed(run, reps, 2, 1)
    assert dstat.item() == 0
    n = sum(c.proj.n * c.proj.k for c in cases)
    nbytes = (n * (0.5 + 1 / 64 + 2) + 4 * sum(o.c2.numel() + 1 for o in outs)
              + 2 * sum(c.A.numel() + c.B.numel() for c in cases))
    return {"weights": n, "ms": ms, "GB/s": nbytes / ms / 1e6, "bytes": nbytes, "out": "bf16"}


# ---------------------------------------------------------------------------
# CPU oracle baseline
# ---------------------------------------------------------------------------

def bench_stack(steps=2, warmup=1, layers=32, M=M_TOKENS, device="cuda"):
    """The 32-layer chained stack of the 7B layer's projections at 8192 tokens
    (r = 16, alpha = 32, weights with 0.1% x10 outliers), both phases:

    * quantize: one batched quantize + DQ call over all 224 fp32 weights
      (6.98 G values), inputs resident in HBM, 4.5159 algorithmic B/weight;
    * fwd+bwd: per layer q = Q(h), k = K(h), v = V(h), a = O(q), g = G(a),
      u = U(a), h' = D(g + u), then the backward through the same graph
      (dh = dX_q + dX_k + dX_v and da = dX_g + dX_u through the accumulate
      flag; k, v and the top take seeded upstream gradients), 32 x 7.211
      TFLOP per pass.  g + u is one torch add (model plumbing, not the method).
    """
    r, s = R, 32.0 / R
    Q, K_, V, O, G, U, D = range(7)
    projs = workloads.LAYER7B
    Ws, outs, adapters = [], [], []
    for layer in range(layers):
        As, Bs = [], []
        for t in range(7):
            W, A, B = workloads.stack_projection(layer, t, device=device)
            Ws.append(W)
            As.append(A)
            Bs.append(B)
            outs.append(binding.NF4Weight.empty(projs[t].n, projs[t].k, device=device))
        adapters.append((As, Bs))
    del W
    qws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device=device)
    dstat = torch.zeros(1, dtype=torch.int32, device=device)
    n_weights = sum(p.n * p.k for p in projs) * layers
    q_ms = timed(lambda: binding.qlora_nf4_quantize_batched(Ws, outs, qws, d_status=dstat), steps, warmup, 1)
    assert dstat.item() == 0, "quantize reported non-finite input"
    q_bytes = n_weights * (4 + 0.5 + 1 / 64) + 4 * sum(o.c2.numel() + 1 for o in outs)
    del Ws
    if device == "cuda":
        torch.cuda.empty_cache()

    ws = torch.empty(max(binding.qlora_linear_ws_bytes(M, p.n, p.k, r) for p in projs), dtype=torch.uint8,
                     device=device)
    binding.qlora_workspace_reset(ws)
    bf = lambda n: torch.empty((M, n), dtype=torch.bfloat16, device=device)  # noqa: E731
    f32 = lambda: torch.empty((M, r), dtype=torch.float32, device=device)  # noqa: E731
    h0 = workloads.stack_input(M, device=device)
    top = workloads.stack_leaf_grad(layers - 1, "top", M, device=device)
    leaf = {(layer, n): workloads.stack_leaf_grad(layer, n, M, device=device)
            for layer in range(layers) for n in ("k", "v")}
    act = [dict(q=bf(4096), k=bf(1024), v=bf(1024), a=bf(4096), g=bf(14336), u=bf(14336), gu=bf(14336),
                out=bf(4096), U=[f32() for _ in range(7)]) for _ in range(layers)]
    grads = [(torch.empty((r, p.k), dtype=torch.float32, device=device),
              torch.empty((p.n, r), dtype=torch.float32, device=device)) for p in projs]
    dgu, da, dq = bf(14336), bf(4096), bf(4096)
    dh_bufs = [bf(4096), bf(4096)]

    def fwd(layer, t, x, y):
        A, B = adapters[layer][0][t], adapters[layer][1][t]
        binding.qlora_linear_fwd(outs[layer * 7 + t], x, A, B, r, s, y, act[layer]["U"][t], ws)

    def bwd(layer, t, x, dy, dx, accumulate):
        A, B = adapters[layer][0][t], adapters[layer][1][t]
        dA, dB = grads[t]
        binding.qlora_linear_bwd(outs[layer * 7 + t], x, dy, A, B, r, s, dx, accumulate, dA, dB, ws,
                                 U=act[layer]["U"][t])

    def step():
        h = h0
        for layer in range(layers):
            a_ = act[layer]
            fwd(layer, Q, h, a_["q"])
            fwd(layer, K_, h, a_["k"])
            fwd(layer, V, h, a_["v"])
            fwd(layer, O, a_["q"], a_["a"])
            fwd(layer, G, a_["a"], a_["g"])
            fwd(layer, U, a_["a"], a_["u"])
            torch.add(a_["g"], a_["u"], out=a_["gu"])
            fwd(layer, D, a_["gu"], a_["out"])
            h = a_["out"]
        dh = top
        for layer in reversed(range(layers)):
            a_ = act[layer]
            x_in = h0 if layer == 0 else act[layer - 1]["out"]
            bwd(layer, D, a_["gu"], dh, dgu, 0)
            bwd(layer, G, a_["a"], dgu, da, 0)
            bwd(layer, U, a_["a"], dgu, da, 1)
            bwd(layer, O, a_["q"], da, dq, 0)
            dh_prev = dh_bufs[layer % 2]
            bwd(layer, Q, x_in, dq, dh_prev, 0)
            bwd(layer, K_, x_in, leaf[(layer, "k")], dh_prev, 1)
            bwd(layer, V, x_in, leaf[(layer, "v")], dh_prev, 1)
            dh = dh_prev

    f_ms = timed(step, steps, warmup, 1)
    assert binding.qlora_workspace_status(ws) == 0, "device status"
    flops = step_flops(M) * layers
    return {
        "quantize": {"weights": n_weights, "ms": q_ms, "GB/s": q_bytes / q_ms / 1e6, "bytes_per_weight": 4.5159},
        "fwd_bwd": {"flops": flops, "ms": f_ms, "TFLOP/s": flops / (f_ms / 1e3) / 1e12},
        "steps": steps, "warmup": warmup,
    }


def oracle_sample_step(cases_cpu, row_div: int, tokens: int):
    """Run the oracle on a bounded sample of the layer step and extrapolate.

    Sample: for each projection, quantize + double-quantize + dequantize the
    first N/row_div rows of the weight, and run the fp64 LoRA forward and
    backward of `tokens` tokens against that slice.  Each part's time is
    scaled by the fraction of the full step's work it represents.
    """
    from oracle import lora, nf4

    t_quant = 0.0
    t_lora = 0.0
    lora_flops = 0.0
    for c in cases_cpu:
        n_rows = max(8, c.proj.n // row_div)
        W = c["W"][:n_rows]
        t0 = time.perf_counter()
        st = nf4.quantize_weight(W)
        Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
        t_quant += (time.perf_counter() - t0) * (c.proj.n / n_rows)
        X, dY, A, B = c["X"][:tokens], c["dY"][:tokens, :n_rows], c["A"], c["B"][:n_rows]
        t0 = time.perf_counter()
        lora.lora_forward(X, Wh, A, B, c.s)
        lora.lora_backward(X, dY, Wh, A, B, c.s)
        dt = time.perf_counter() - t0
        f_sample = 4 * tokens * n_rows * c.proj.k + 6 * tokens * R * (n_rows + c.proj.k)
        f_full = 4 * M_TOKENS * c.proj.n * c.proj.k + 6 * M_TOKENS * R * (c.proj.n + c.proj.k)
        t_lora += dt * f_full / f_sample
        lora_flops += f_sample
    total = t_quant + t_lora
    return step_flops() / total / 1e12, total


def oracle_secondary(device, row_div=16):
    """The oracle on bounded samples of the secondary rows, times scaled to
    the full work (rank 0, N = 1, beside the GPU's own rows):

    * quantize + DQ and dequantize (bf16) of the first N/row_div rows of each
      of the six tensors of the first OPT-1.3B layer, as weights/s and GB/s at
      4.5159 and 2.5159 algorithmic bytes per weight;
    * the decode-shaped forward on the 14336 x 4096 gate at M = 16: fp32
      decode of the first N/row_div rows plus the fp64 forward of those rows
      (the sample's quantization is not timed), as microseconds per full call.
    """
    from oracle import lora, nf4

    t_q = t_d = 0.0
    n = 0
    for layer, t, p in workloads.opt13b_weight_shapes():
        if layer != 0:
            continue
        rows = max(8, p.n // row_div)
        W = workloads.opt13b_weight(layer, t, device=device)[:rows].cpu().numpy()
        t0 = time.perf_counter()
        st = nf4.quantize_weight(W)
        t1 = time.perf_counter()
        nf4.dequantize_weight(st, "bf16")
        t2 = time.perf_counter()
        t_q += t1 - t0
        t_d += t2 - t1
        n += rows * p.k
    case = workloads.gemv_case(16, device=device)
    rows = max(8, case.proj.n // row_div)
    st = nf4.quantize_weight(case.W[:rows].cpu().numpy())
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
    X, A, B = f64(case.X), f64(case.A), f64(case.B[:rows])
    t0 = time.perf_counter()
    Wh = nf4.dequantize_weight(st, "fp32").astype(np.float64)
    lora.lora_forward(X, Wh, A, B, case.s)
    t_gemv = (time.perf_counter() - t0) * (case.proj.n / rows)
    return {
        "quantize": {"weights_per_s": n / t_q, "GB/s": n * 4.5159 / t_q / 1e9},
        "dequant_bf16": {"weights_per_s": n / t_d, "GB/s": n * 2.5159 / t_d / 1e9},
        "gemv_gate_14336x4096_M16": {"us_per_call": t_gemv * 1e6},
        "sample": (f"first 1/{row_div} of the rows of the first OPT-1.3B layer's six tensors ({n} weights); "
                   f"first 1/{row_div} of the gate's rows at M = 16; times scaled to full calls"),
    }


class CpuCase(dict):
    """Host copies of one projection's inputs (first `tokens` token rows only)."""

    def __init__(self, case, tokens):
        f64 = lambda t: t.float().cpu().numpy().astype(np.float64)  # noqa: E731
        super().__init__(W=case.W.cpu().numpy(), X=f64(case.X[:tokens]), dY=f64(case.dY[:tokens]),
                         A=f64(case.A), B=f64(case.B))
        self.proj = case.proj
        self.s = case.s


def cpu_cases(device, tokens):
    return [CpuCase(workloads.layer7b_case(t, m=M_TOKENS, device=device), tokens) for t in range(7)]


def cpu_model() -> str:
    """The host CPU's model name (from /proc/cpuinfo), or the platform's processor string."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform

    return platform.processor() or "unknown"


def cores_used():
    try:
        return len(os.sched_getaffinity(0))
    except AttributeError:
        return os.cpu_count()


# ---------------------------------------------------------------------------
# Arms
# ---------------------------------------------------------------------------

def run_reference(args, rank, world):
    if rank != 0:
        return
    row_div, tokens = 256, 32
    cases = cpu_cases("cuda" if torch.cuda.is_available() else "cpu", tokens)
    for _ in range(args.warmup):
        oracle_sample_step(cases, row_div, tokens)
    vals = []
    t0 = time.perf_counter()
    for _ in range(args.steps):
        v, _ = oracle_sample_step(cases, row_div, tokens)
        vals.append(v)
    wall = time.perf_counter() - t0
    value = statistics.median(vals)
    sample = (f"oracle (numpy, fp64 LoRA) on 1/{row_div} of each weight's rows and {tokens} of {M_TOKENS} tokens "
              f"per projection, times scaled to the full step")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_flops() / (value * 1e12) * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": WORKLOAD, "flops_per_step_per_gpu": step_flops(), "parallelism": "replicas x1"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle", "sample": sample,
                         "cpu_model": cpu_model(), "nproc": os.cpu_count()},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "wall_s": wall,
    }))


GEMM_TRAFFIC_PROFILE = os.path.join(ROOT, "profiles", "gemm_nf4_layer_step_traffic.md")
GEMM_SOURCES = ("csrc/gemm_nf4.cu", "csrc/gemm_common.cuh", "csrc/common.cuh")  # the GEMM and its device helpers


def gemm_traffic_per_launch():
    """DRAM bytes per gemm_nf4 launch from the committed ncu summary, or None
    when the kernel's sources changed since that capture."""
    import hashlib
    try:
        text = open(GEMM_TRAFFIC_PROFILE).read()
    except OSError:
        return None
    fields = dict(line.split(": ", 1) for line in text.splitlines()
                  if line.startswith(("traffic_bytes_per_launch: ", "source_digest: ")))
    h = hashlib.sha256()
    for rel in GEMM_SOURCES:
        with open(os.path.join(ROOT, "bit_nf4_quantized_blk_b200", rel), "rb") as f:
            h.update(f.read())
    if fields.get("source_digest", "").strip() != h.hexdigest()[:16]:
        return None
    return int(fields["traffic_bytes_per_launch"])


def run_ours(args, rank, world, local_rank):
    from bit_nf4_quantized_blk_b200 import build

    build.build()
    device = "cuda"
    peaks, peak_src = load_peaks()
    step = LayerStep(device)
    step.run()
    torch.cuda.synchronize()
    step.check_status()

    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    smi_index = int(vis.split(",")[local_rank]) if vis and vis.split(",")[0].isdigit() else local_rank
    clock = ClockSampler(smi_index)
    binding.qlora_timing_enable(True)
    clock.start()
    window = []
    ms = timed(step.run if args.streams == 1 else step.run_two_streams, args.steps, args.warmup, world, window)
    clocks = clock.stop(window)
    fam = {f: binding.qlora_timing_read(f) for f in ("quantize", "dequant", "gemv", "side", "gemm")}
    binding.qlora_timing_enable(False)
    step.check_status()
    launches_total = sum(n for _, n in fam.values())
    steps_recorded = args.steps + args.warmup
    gemm_ms, gemm_n = fam["gemm"]
    gemm_ms_per_step = gemm_ms / steps_recorded
    gemm_tflops = gemm_flops_per_step() / (gemm_ms_per_step / 1e3) / 1e12
    # The timed region is a fraction of a second at full clock: the burst
    # cuBLAS figure is the comparable peak.  The clock-normalised fraction
    # divides by the peak scaled to the median SM clock sampled in the timed
    # region (the burst figure taken as a 1965 MHz one unless the peaks file
    # records its clock).
    peak = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    peak_mhz = next((float(v) for k, v in peaks.items() if "bf16" in k and "mhz" in k and "sustained" not in k
                     and isinstance(v, (int, float))), 1965.0)
    frac_clock = (gemm_tflops / (peak * clocks["sm_mhz"] / peak_mhz)
                  if clocks and clocks.get("sm_mhz") else None)

    flops = step_flops()
    value = job_throughput(flops, world, ms) / 1e12

    # end-to-end through host buffers
    h2d, d2h = step.host_buffers()
    e2e_ms = step.e2e_timed(max(4, args.steps // 4), 2, world)
    e2e_value = job_throughput(flops, world, e2e_ms) / 1e12

    line = {
        "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": WORKLOAD,
                   "flops_per_step_per_gpu": flops, "l2": "inputs larger than L2 (GBs per step)",
                   "parallelism": f"replicas x{world}",
                   **({"streams": "projections alternate over 2 streams"} if args.streams == 2 else {})},
        "roofline": {"bound": "tensor",
                     "kernel": "gemm_nf4_kernel (tcgen05 pair-CTA 512x256 tile, 4-bit weight decoded into shared memory)",
                     "achieved": gemm_tflops, "peak": peak, "unit": "TFLOP/s", "frac": gemm_tflops / peak,
                     "peak_source": f"{peak_src} bf16_tflops (burst; the timed region is "
                                    f"{args.steps * ms / 1e3:.2f} s at the sampled clock)",
                     "frac_clock_normalized": frac_clock, "peak_clock_mhz": peak_mhz,
                     "traffic": gemm_traffic_per_launch(),
                     "traffic_unit": "bytes per launch (ncu dram read + write)",
                     "share_of_step": gemm_ms_per_step / ms,
                     "gemm_ms_per_step": gemm_ms_per_step, "gemm_flops_per_step": gemm_flops_per_step()},
        "gpu_launches": int(round(launches_total / steps_recorded * args.steps)),
        "kernel_ms_per_step": {f: v[0] / steps_recorded for f, v in fam.items()},
        "clocks": clocks,
        "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                "ms_per_step": e2e_ms,
                "pipeline": "every step uploads its inputs and downloads its outputs; step i+1's upload and "
                            "step i-1's download overlap step i's compute (3 streams, 2 device buffer sets)"},
    }
    if rank == 0 and not args.no_extras:
        del step
        torch.cuda.empty_cache()
        extras = bench_quantize_dequant(clock=smi_index)
        extras["gemv_gate_14336x4096"] = bench_gemv()
        extras["merge_layer7b_r16"] = bench_merge()
        hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        for k in ("quantize", "dequant_bf16", "merge_layer7b_r16"):
            extras[k]["frac_hbm"] = extras[k]["GB/s"] / hbm
        for k, v in extras["gemv_gate_14336x4096"].items():
            if isinstance(v, dict):
                v["frac_hbm"] = v["GB/s"] / hbm
                v["write_flush"]["frac_hbm"] = v["write_flush"]["GB/s"] / hbm
        extras["hbm_peak_gbs"] = hbm
        line["secondary"] = extras
    if rank == 0 and not args.no_stack:
        torch.cuda.empty_cache()
        st, st_clocks = ClockSampler.around(smi_index, bench_stack)
        line.setdefault("secondary", {})["stack_32x7_8192tok"] = st
        st["clocks"] = st_clocks
        st["quantize"]["frac_hbm"] = st["quantize"]["GB/s"] / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
        st["fwd_bwd"]["frac_bf16_burst"] = st["fwd_bwd"]["TFLOP/s"] / peak
        st["fwd_bwd"]["frac_bf16_sustained"] = st["fwd_bwd"]["TFLOP/s"] / peaks.get(
            "bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"])
    if rank == 0 and world == 1 and not args.no_cpu:
        cases = cpu_cases(device, 256)
        v, t = oracle_sample_step(cases, 32, 256)
        line["cpu_baseline"] = {"value": v, "unit": "TFLOP/s", "cores": cores_used(), "kind": "oracle",
                                "cpu_model": cpu_model(), "nproc": os.cpu_count(),
                                "sample": "oracle (numpy; fp64 LoRA) on 1/32 of each weight's rows and 256 of 8192 "
                                          "tokens per projection, times scaled to the full step",
                                "extrapolated_step_s": t,
                                "secondary": oracle_secondary(device)}
    if rank == 0:
        print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-extras", action="store_true")
    ap.add_argument("--no-cpu", action="store_true")
    ap.add_argument("--streams", type=int, choices=[1, 2], default=1,
                    help="2: the timed step alternates the projections' calls over two streams")
    ap.add_argument("--no-stack", action="store_true",
                    help="skip the 32-layer chained stack (quantize, fwd+bwd; about 35 GB on the device), "
                         "which the default run times on rank 0")
    args = ap.parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local_rank)
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=300))
    if args.impl == "reference":
        run_reference(args, rank, world)
    else:
        run_ours(args, rank, world, local_rank)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
