"""GPU parity: quantize + double quantize + dequantize are bit-exact with the oracle.

Everything is called through the C ABI (ctypes binding); expected values come
only from ``oracle/`` on the same seeded inputs.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_state_equal, f32_bits, gpu_quantize, require_gpu
from oracle import nf4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _check_dequant(out, st, shape):
    rows, cols = shape
    y16 = torch.empty((rows, cols), dtype=torch.bfloat16, device="cuda")
    binding.qlora_nf4_dequantize(out, y16, 0, 0)
    y32 = torch.empty((rows, cols), dtype=torch.float32, device="cuda")
    binding.qlora_nf4_dequantize(out, y32, 1, 0)
    yt = torch.empty((cols, rows), dtype=torch.bfloat16, device="cuda")
    if rows % 8 == 0:
        binding.qlora_nf4_dequantize(out, yt, 0, 1)
    torch.cuda.synchronize()
    want32 = nf4.dequantize_weight(st, "fp32")
    want16 = nf4.dequantize_weight(st, "bf16")
    assert np.array_equal(f32_bits(y32.cpu().numpy()), f32_bits(want32)), "fp32 dequant differs"
    got16 = y16.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got16, want16), "bf16 dequant differs"
    if rows % 8 == 0:
        gott = yt.view(torch.int16).cpu().numpy().view(np.uint16)
        assert np.array_equal(gott, want16.T), "transposed bf16 dequant differs"


def test_tiny_config_bit_exact():
    case = workloads.tiny_case()
    st = nf4.quantize_weight(case.W.numpy())
    out = gpu_quantize(case.W)
    assert_state_equal(out, st, "tiny")
    assert np.all(out.packed[:32].cpu().numpy() == 0x77)  # the zeroed block
    _check_dequant(out, st, (1024, 1024))


@pytest.mark.parametrize("shape", [(1, 64), (3, 192), (5, 4160), (257, 128), (8, 16384 + 64), (64, 64 * 257)])
def test_ragged_shapes_bit_exact(shape):
    rows, cols = shape
    W = workloads.normal_f32(shape, 0.02, 100 + rows)
    W[rows // 2, :64] = 0.0  # a zero block in the middle
    st = nf4.quantize_weight(W.numpy())
    out = gpu_quantize(W)
    assert_state_equal(out, st, str(shape))
    _check_dequant(out, st, shape)


def test_edge_values_bit_exact():
    # Blocks of absmax 1 holding every threshold, its predecessor, every level,
    # +-0 and subnormals; blocks of subnormal absmax; a block of -0.0.
    T = nf4.decision_thresholds()
    vals = np.concatenate([T, np.nextafter(T, np.float32(-2)), nf4.NF4_LEVELS,
                           np.array([0.0, -0.0, 1e-45, -1e-45, 1e-39, -3e-39], np.float32)])
    rows = []
    for s in range(0, vals.size, 63):
        blk = np.zeros(64, np.float32)
        chunk = vals[s:s + 63]
        blk[:chunk.size] = chunk
        blk[63] = 1.0
        rows.append(blk)
    sub = np.zeros(64, np.float32)
    sub[:6] = np.array([1e-45, -2e-45, 3e-45, 1e-41, -1e-41, 7e-42], np.float32)
    rows.append(sub)
    rows.append(np.full(64, -0.0, np.float32))
    rows.append(np.linspace(-3.0, 3.0, 64, dtype=np.float32))
    W = np.stack(rows + [rows[0]] * ((8 - len(rows) % 8) % 8)).astype(np.float32)
    st = nf4.quantize_weight(W)
    out = gpu_quantize(torch.from_numpy(W))
    assert_state_equal(out, st, "edge values")
    _check_dequant(out, st, W.shape)


def test_wide_exponent_spread_uses_the_sequential_mean():
    # Block scales spanning ~2^-100 .. 2^10: the fp64 sum is not exact in every
    # order here, so the kernels must take the sequential path of the definition.
    rng = np.random.default_rng(7)
    rows, cols = 64, 64 * 300
    W = rng.normal(0, 1, (rows, cols)).astype(np.float32)
    scales = np.exp2(rng.uniform(-100, 10, rows * cols // 64)).astype(np.float32)
    W = (W.reshape(-1, 64) * scales[:, None]).astype(np.float32).reshape(rows, cols)
    st = nf4.quantize_weight(W)
    out = gpu_quantize(torch.from_numpy(W))
    assert_state_equal(out, st, "wide spread")


def test_nonfinite_input_is_reported():
    W = workloads.normal_f32((8, 128), 0.02, 5)
    W[3, 17] = float("nan")
    with pytest.raises(binding.QloraError) as e:
        gpu_quantize(W)
    assert e.value.status == 3
    W[3, 17] = float("inf")
    out = binding.NF4Weight.empty(8, 128)
    ws = torch.empty(binding.qlora_nf4_sizes(8, 128)["ws_bytes"], dtype=torch.uint8, device="cuda")
    d_status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    binding.qlora_nf4_quantize(W.cuda(), out, ws, d_status=d_status)
    torch.cuda.synchronize()
    assert d_status.item() == 3
    W[3, 17] = 0.5
    binding.qlora_nf4_quantize(W.cuda(), out, ws, d_status=d_status)
    torch.cuda.synchronize()
    assert d_status.item() == 0


def test_batched_equals_per_tensor():
    shapes = [(64, 128), (3, 192), (128, 4096), (1, 64), (200, 320)]
    Ws = [workloads.normal_f32(s, 0.02, 40 + i) for i, s in enumerate(shapes)]
    outs = [binding.NF4Weight.empty(*s) for s in shapes]
    ws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize_batched([w.cuda() for w in Ws], outs, ws)
    for W, out, s in zip(Ws, outs, shapes):
        assert_state_equal(out, nf4.quantize_weight(W.numpy()), f"batched {s}")
    ys = [torch.empty(s, dtype=torch.bfloat16, device="cuda") for s in shapes]
    binding.qlora_nf4_dequantize_batched(outs, ys, 0)
    torch.cuda.synchronize()
    for W, y, s in zip(Ws, ys, shapes):
        want = nf4.dequantize_weight(nf4.quantize_weight(W.numpy()), "bf16")
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want), f"batched dequant {s}"


def test_opt13b_shapes_full_batch():
    """Quantize + DQ over the 168 OPT-1.3B-shaped tensors (1.208 G weights,
    0.1% outliers) in one batched call, the launch the bench times; check the
    first and last layers' tensors bit for bit against the oracle."""
    items = workloads.opt13b_weight_shapes()
    Ws = [workloads.opt13b_weight(layer, t, device="cuda") for layer, t, _ in items]
    outs = [binding.NF4Weight.empty(p.n, p.k) for _, _, p in items]
    ws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize_batched(Ws, outs, ws)
    torch.cuda.synchronize()
    check = [i for i, (layer, t, _) in enumerate(items) if layer in (0, 23)]
    for i in check:
        layer, t, p = items[i]
        st = nf4.quantize_weight(Ws[i].cpu().numpy())
        assert_state_equal(outs[i], st, f"layer {layer} {p.name}")
    ys = [torch.empty((p.n, p.k), dtype=torch.bfloat16, device="cuda") for _, _, p in items]
    binding.qlora_nf4_dequantize_batched(outs, ys, 0)
    torch.cuda.synchronize()
    for i in check[:3]:
        st = nf4.quantize_weight(Ws[i].cpu().numpy())
        want = nf4.dequantize_weight(st, "bf16")
        assert np.array_equal(ys[i].view(torch.int16).cpu().numpy().view(np.uint16), want)
