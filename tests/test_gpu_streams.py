"""GPU: calls overlapping on two streams give the serial results bit for bit.

The seven projections of the 7B layer step at 8192 tokens run once serially
on one stream, then with their forward and backward calls alternating over
two streams, each stream with its own workspace, so that one projection's
HBM-bound rank-r kernels overlap another's GEMM.  Each output (Y, dX, dA, dB)
must be bit-identical to the serial run's: every kernel sums in a fixed
order, so overlap may change timing but never a result.  The same
comparison with a 650 MB fill kernel before every call changes the timing
of the serial step.
"""

import pytest
import torch

import bench
from bit_nf4_quantized_blk_b200 import binding
from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def step():
    require_gpu()
    torch.cuda.set_device(0)
    return bench.LayerStep("cuda")


def _outputs(step):
    return [t.clone() for t in step.Y + step.dX + step.dA + step.dB]


def _names():
    return [f"{k}[{i}]" for k in ("Y", "dX", "dA", "dB") for i in range(7)]


def _differing(a, b):
    bits = lambda t: t.view(torch.int32) if t.dtype == torch.float32 else t.view(torch.int16)  # noqa: E731
    return [n for n, x, y in zip(_names(), a, b) if not torch.equal(bits(x), bits(y))]


def _serial(step):
    step.run()
    torch.cuda.synchronize()
    return _outputs(step)


def _two_streams(step, wss, streams):
    main = torch.cuda.current_stream()
    binding.qlora_nf4_quantize_batched([c.W for c in step.cases], step.outs, step.qws, d_status=step.dstat)
    for st in streams:
        st.wait_stream(main)
    fwd_done = []
    for i, (c, o, Y, U) in enumerate(zip(step.cases, step.outs, step.Y, step.U)):
        st = streams[i % 2]
        with torch.cuda.stream(st):
            binding.qlora_linear_fwd(o, c.X, c.A, c.B, c.r, c.s, Y, U, wss[i % 2])
            ev = torch.cuda.Event()
            ev.record(st)
            fwd_done.append(ev)
    for j, i in enumerate(reversed(range(7))):
        c, o = step.cases[i], step.outs[i]
        st = streams[j % 2]
        with torch.cuda.stream(st):
            st.wait_event(fwd_done[i])  # U of projection i
            binding.qlora_linear_bwd(o, c.X, c.dY, c.A, c.B, c.r, c.s, step.dX[i], 0, step.dA[i], step.dB[i],
                                     wss[j % 2], U=step.U[i])
    for st in streams:
        main.wait_stream(st)
    torch.cuda.synchronize()
    return _outputs(step)


def _serial_with_fills(step, fill):
    binding.qlora_nf4_quantize_batched([c.W for c in step.cases], step.outs, step.qws, d_status=step.dstat)
    for c, o, Y, U in zip(step.cases, step.outs, step.Y, step.U):
        fill.fill_(1.0)
        binding.qlora_linear_fwd(o, c.X, c.A, c.B, c.r, c.s, Y, U, step.lws)
    for c, o, dX, dA, dB, U in reversed(list(zip(step.cases, step.outs, step.dX, step.dA, step.dB, step.U))):
        fill.fill_(2.0)
        binding.qlora_linear_bwd(o, c.X, c.dY, c.A, c.B, c.r, c.s, dX, 0, dA, dB, step.lws, U=U)
    torch.cuda.synchronize()
    return _outputs(step)


def test_two_streams_match_serial_bit_for_bit(step):
    ref = _serial(step)
    assert _differing(ref, _serial(step)) == []
    ws2 = torch.empty_like(step.lws)
    binding.qlora_workspace_reset(ws2)
    wss = [step.lws, ws2]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for trial in range(8):
        assert _differing(ref, _two_streams(step, wss, streams)) == [], f"trial {trial}"
    assert [binding.qlora_workspace_status(w) for w in wss] == [0, 0]
    assert step.dstat.item() == 0


def test_fill_kernels_between_calls_change_nothing(step):
    ref = _serial(step)
    fill = torch.empty(650 * 2**20 // 4, dtype=torch.float32, device="cuda")
    for trial in range(2):
        assert _differing(ref, _serial_with_fills(step, fill)) == [], f"trial {trial}"
    del fill


def test_bench_two_stream_step_matches_serial(step):
    """bench.py --streams 2 times LayerStep.run_two_streams: its outputs equal
    the serial step's bit for bit, and neither workspace records a device error."""
    ref = _serial(step)
    for trial in range(3):
        step.run_two_streams()
        torch.cuda.synchronize()
        assert _differing(ref, _outputs(step)) == [], f"trial {trial}"
    step.check_status()
