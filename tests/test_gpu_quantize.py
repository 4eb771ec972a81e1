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


def test_dq_rounding_ties_bit_exact():
    """Block scales whose deviations land exactly on rounding ties of the
    int8 scale codes (a chunk of 256 scales 256 +- d, d = 127 and every
    k + 1/2): the kernel rounds them to even like the oracle (0.5 -> 0,
    1.5 -> 2, 2.5 -> 2).  Each block's absmax is its first weight, with either
    sign; the other weights are smaller random values."""
    d = np.array([127.0] + [k + 0.5 for k in range(127)], np.float32)
    a = np.empty(256, np.float32)
    a[0::2] = np.float32(256.0) + d
    a[1::2] = np.float32(256.0) - d
    rng = np.random.default_rng(41)
    W = (rng.uniform(-0.9, 0.9, (256, 64)) * a[:, None]).astype(np.float32)
    W[:, 0] = a * np.where(np.arange(256) % 3 == 0, -1.0, 1.0).astype(np.float32)
    st = nf4.quantize_weight(W)
    assert st.mu == np.float32(256.0) and st.c2[0] == np.float32(127.0)
    out = gpu_quantize(torch.from_numpy(W))
    assert_state_equal(out, st, "DQ ties")
    q = out.qscale.cpu().numpy()
    assert [int(v) for v in q[2:8]] == [0, 0, 2, -2, 2, -2]


def _adversarial_absmax(rng) -> np.ndarray:
    """Block absmax values away from 1: log-uniform random ones over most of
    the fp32 range, the fp32 neighbours of powers of two, values around both
    ends of the kernel's reciprocal fast range (2^-121 and 2^119), subnormal
    and tiny ones (the IEEE-division path), and the largest finite values."""
    f = np.float32
    vals = list((2.0 ** rng.uniform(-120.0, 118.0, 1500)).astype(f))
    for e in rng.integers(-125, 127, 200):
        p = f(2.0 ** int(e))
        vals += [np.nextafter(p, f(0)), p, np.nextafter(p, f(np.inf)), f(p * f(1.0 + 3 * 2.0 ** -23))]
    for edge in (f(2.0 ** -121), f(2.0 ** 119)):
        x = edge
        for _ in range(12):
            x = np.nextafter(x, f(0))
        for _ in range(25):
            vals.append(x)
            x = np.nextafter(x, f(np.inf))
        vals += list((edge * (1.0 + rng.uniform(-0.01, 0.01, 40))).astype(f))
    vals += [f(2.0 ** -130), f(2.0 ** -140), f(7 * 2.0 ** -149), f(3e38), np.finfo(f).max, f(2.0 ** -126)]
    a = np.array(vals, dtype=f)
    return a[(a > 0) & np.isfinite(a)]


def _adversarial_weight(codebook: str, seed: int) -> np.ndarray:
    """Blocks whose weights sit on the kernel's decision edges for their block
    absmax a (one weight of magnitude a, random sign and position, per
    block): fl32(T_j a) and its fp32 neighbours up to 3 ulps either side, and
    fl32(T_j a (1 +- 2^-19)) +- 1 ulp, the edges of the band inside which the
    kernel recodes from the IEEE quotient.  Blocks are padded with uniform
    weights in (-a, a)."""
    f = np.float32
    rng = np.random.default_rng(seed)
    T = nf4.decision_thresholds(codebook).astype(np.float64)
    blocks = []
    for a in _adversarial_absmax(rng):
        cand = []
        for t in T:
            c = f(t * float(a))
            lo = hi = c
            cand.append(c)
            for _ in range(3):
                lo, hi = np.nextafter(lo, f(-np.inf)), np.nextafter(hi, f(np.inf))
                cand += [lo, hi]
            for rel in (1.0 - 2.0 ** -19, 1.0 + 2.0 ** -19):
                e = f(t * float(a) * rel)
                cand += [np.nextafter(e, f(-np.inf)), e, np.nextafter(e, f(np.inf))]
        cand = np.array(cand, dtype=f)
        cand = cand[np.abs(cand) <= a]
        per = 63
        nb = -(-cand.size // per)
        pad = (rng.uniform(-1.0, 1.0, nb * per - cand.size) * float(a)).astype(f)
        body = np.concatenate([cand, pad]).reshape(nb, per)
        for row in body:
            pos = int(rng.integers(0, 64))
            sign = f(-1.0) if rng.integers(0, 2) else f(1.0)
            blocks.append(np.insert(row, pos, sign * a))
    W = np.stack(blocks).astype(f)
    assert np.isfinite(W).all()
    return W


@pytest.mark.parametrize("codebook,scales", [("nf4", "dq_int8"), ("fp4", "dq_int8"), ("nf4", "fp32")])
def test_decision_edges_at_block_scales_away_from_one(codebook, scales):
    """Bit-exact codes (and the rest of the state) where the reciprocal fast
    path is closest to being wrong: the block absmax is not a power of two
    (or sits at the ends of the fast range) and the weights lie on and next
    to every decision threshold and band edge."""
    W = _adversarial_weight(codebook, 17 if codebook == "nf4" else 18)
    # self-check of the construction: many weights normalise to within 2 ulps of a threshold
    a = np.abs(W).max(axis=1, keepdims=True)
    x = (W / a).astype(np.float32)
    T = nf4.decision_thresholds(codebook)
    near = np.zeros(x.shape, bool)
    for t in T:
        near |= np.abs(x.astype(np.float64) - float(t)) <= 2.0 * float(np.spacing(np.float32(abs(t))))
    assert near.sum() > 100_000 if codebook == "nf4" else near.sum() > 50_000
    cb = binding.CODEBOOK_NF4 if codebook == "nf4" else binding.CODEBOOK_FP4
    sf = binding.SCALES_DQ_INT8 if scales == "dq_int8" else binding.SCALES_FP32
    st = nf4.quantize_weight(W, codebook=codebook, scale_format=scales)
    out = gpu_quantize(torch.from_numpy(W), cb, sf)
    assert_state_equal(out, st, f"decision edges {codebook} {scales}")
