"""GPU parity of the stored-format variants against the oracle.

Codebooks NF4 and FP4 ("FT-02: QLoRA -- Fine-Tuning with Quantization",
"Exercise 3: NF4 vs FP4 at equal memory"); block scales as int8 or E4M3
double-quantized codes or plain fp32 ("QLoRA Deep Dive ...", section "2.
Squeezing More Memory: Double Quantization (DQ)"); fp32, bf16 and fp16 input
weights.  Codes, scale codes and dequantized weights are bit-exact; linear
layer and merge outputs meet the float tolerance of the other parity tests.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, assert_state_equal, bf16_to_np, f32_bits, gpu_quantize, require_gpu, workspace
from oracle import lora, nf4

pytestmark = pytest.mark.gpu

CB = {"nf4": binding.CODEBOOK_NF4, "fp4": binding.CODEBOOK_FP4}
SF = {"dq_int8": binding.SCALES_DQ_INT8, "dq_fp8": binding.SCALES_DQ_FP8, "fp32": binding.SCALES_FP32}
FORMATS = [(c, f) for c in CB for f in SF]


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _weights(shape, seed):
    W = workloads.normal_f32(shape, 0.02, seed)
    workloads.with_outliers(W, seed)
    W.view(-1)[:64] = 0.0  # one all-zero block
    return W


@pytest.mark.parametrize("codebook,fmt", FORMATS)
@pytest.mark.parametrize("shape", [(1024, 1024), (3, 64), (37, 192), (5, 16448)])
def test_quantize_bit_exact(codebook, fmt, shape):
    W = _weights(shape, 40 + shape[0])
    st = nf4.quantize_weight(W.numpy(), codebook=codebook, scale_format=fmt)
    out = gpu_quantize(W, CB[codebook], SF[fmt])
    assert_state_equal(out, st, f"{codebook}/{fmt} {shape}")
    if codebook == "fp4":
        codes = nf4.unpack_nibbles(out.packed.cpu().numpy(), W.numel())
        assert not np.any(codes == 8), "FP4 quantization emitted -0"


@pytest.mark.parametrize("codebook,fmt", FORMATS)
def test_batched_quantize_matches_per_tensor(codebook, fmt):
    shapes = [(64, 256), (7, 64), (130, 1024)]
    Ws = [_weights(s, 70 + i) for i, s in enumerate(shapes)]
    outs = [binding.NF4Weight.empty(r, c, codebook=CB[codebook], scale_format=SF[fmt]) for r, c in shapes]
    ws = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(outs), dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize_batched_ex([w.cuda() for w in Ws], outs, ws)
    for W, o, s in zip(Ws, outs, shapes):
        assert_state_equal(o, nf4.quantize_weight(W.numpy(), codebook=codebook, scale_format=fmt), f"batch {s}")


@pytest.mark.parametrize("dtype,name", [(torch.bfloat16, "bf16"), (torch.float16, "fp16")])
@pytest.mark.parametrize("codebook,fmt", [("nf4", "dq_int8"), ("fp4", "dq_fp8"), ("nf4", "fp32")])
def test_16bit_inputs(dtype, name, codebook, fmt):
    W = _weights((96, 1024), 5).to(dtype)
    if dtype == torch.float16:
        W.view(-1)[64:80] = torch.tensor([6e-8, -6e-8, 3e-5, 65504.0] * 4, dtype=dtype)  # subnormals, max
    bits = W.view(torch.int16).numpy().view(np.uint16)
    st = nf4.quantize_weight(nf4.widen_16bit(bits, name).reshape(W.shape), codebook=codebook, scale_format=fmt)
    out = gpu_quantize(W, CB[codebook], SF[fmt])
    assert_state_equal(out, st, f"{name} {codebook}/{fmt}")


def test_16bit_input_nonfinite_is_reported():
    W = workloads.normal_f32((8, 128), 0.02, 5).to(torch.bfloat16)
    W[3, 7] = float("inf")
    out = binding.NF4Weight.empty(8, 128)
    ws = torch.empty(binding.qlora_nf4_sizes(8, 128)["ws_bytes"], dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.QloraError, match="NONFINITE"):
        binding.qlora_nf4_quantize_ex(W.cuda(), out, ws)


def test_fp8_scale_codes_at_exact_ties_and_subnormals():
    """A single-chunk tensor whose block absmax values are 4 +- 2 x with x
    every positive E4M3 value below 1 and every midpoint between neighbours:
    the mean is exactly 4, c2 exactly 2, so fp32(d / c2) = +-x exactly and
    the E4M3 rounding meets its ties (half to even) and its subnormals."""
    vals = nf4.e4m3_decode(np.arange(0x39, dtype=np.uint8)).astype(np.float64)  # 0 .. 1
    xs = list(vals[1:-1]) + list((vals[:-1] + vals[1:]) / 2)
    xs = xs[:127]
    rng = np.random.default_rng(3)
    while len(xs) < 127:
        xs.append(float(rng.uniform(0, 1)))
    a = [6.0, 2.0] + [4.0 + 2.0 * x for x in xs] + [4.0 - 2.0 * x for x in xs]
    assert len(a) == 256
    W = np.zeros((16, 1024), np.float32)
    for b, ab in enumerate(a):
        row, col = divmod(b * 64, 1024)
        W[row, col] = ab
        W[row, col + 1 : col + 64] = np.float32(ab) * np.linspace(-0.9, 0.9, 63, dtype=np.float32)
    st = nf4.quantize_weight(W, scale_format="dq_fp8")
    assert st.mu == np.float32(4.0) and st.c2[0] == np.float32(2.0)
    out = gpu_quantize(torch.from_numpy(W), binding.CODEBOOK_NF4, binding.SCALES_DQ_FP8)
    assert_state_equal(out, st, "E4M3 ties")


@pytest.mark.parametrize("codebook,fmt", FORMATS)
def test_dequantize_bit_exact(codebook, fmt):
    W = _weights((136, 1024), 9)
    st = nf4.quantize_weight(W.numpy(), codebook=codebook, scale_format=fmt)
    out = gpu_quantize(W, CB[codebook], SF[fmt])
    d32 = torch.empty((136, 1024), dtype=torch.float32, device="cuda")
    d16 = torch.empty((136, 1024), dtype=torch.bfloat16, device="cuda")
    dT = torch.empty((1024, 136), dtype=torch.bfloat16, device="cuda")
    binding.qlora_nf4_dequantize(out, d32, 1)
    binding.qlora_nf4_dequantize(out, d16, 0)
    binding.qlora_nf4_dequantize(out, dT, 0, 1)
    torch.cuda.synchronize()
    ref32 = nf4.dequantize_weight(st, "fp32")
    ref16 = nf4.dequantize_weight(st, "bf16")
    assert np.array_equal(f32_bits(d32.cpu().numpy()), f32_bits(ref32))
    assert np.array_equal(d16.cpu().view(torch.int16).numpy().view(np.uint16), ref16)
    assert np.array_equal(dT.cpu().view(torch.int16).numpy().view(np.uint16), ref16.T)


@pytest.mark.parametrize("codebook,fmt", [("fp4", "dq_fp8"), ("nf4", "fp32"), ("fp4", "fp32"), ("nf4", "dq_fp8")])
@pytest.mark.parametrize("M", [4, 16, 96])
def test_linear_forward_backward(codebook, fmt, M):
    N, K, r, s = 512, 4160, 16, 2.0
    W = _weights((N, K), 11)
    A = workloads.normal_bf16((r, K), 0.02, 12)
    B = workloads.normal_bf16((N, r), 0.02, 13)
    X = workloads.normal_bf16((M, K), 1.0, 14)
    dY = workloads.normal_bf16((M, N), 1.0, 15)
    st = nf4.quantize_weight(W.numpy(), codebook=codebook, scale_format=fmt)
    Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
    out = gpu_quantize(W, CB[codebook], SF[fmt])
    ws = workspace(M, N, K, r)
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, r), dtype=torch.float32, device="cuda")
    Xd, Ad, Bd, dYd = X.cuda(), A.cuda(), B.cuda(), dY.cuda()
    binding.qlora_linear_fwd(out, Xd, Ad, Bd, r, s, Y, U, ws)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    binding.qlora_linear_bwd(out, Xd, dYd, Ad, Bd, r, s, dX, 0, dA, dB, ws, U=U)
    assert binding.qlora_workspace_status(ws) == 0
    Y_ref, U_ref = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    dX_ref, dA_ref, dB_ref, _ = lora.lora_backward(_np(X), _np(dY), Wh, _np(A), _np(B), s)
    assert_close(bf16_to_np(Y), Y_ref, f"Y {codebook}/{fmt} M={M}")
    assert_close(bf16_to_np(dX), dX_ref, f"dX {codebook}/{fmt} M={M}")
    assert_close(_np(dA), dA_ref, "dA")
    assert_close(_np(dB), dB_ref, "dB")


@pytest.mark.parametrize("codebook,fmt", [("fp4", "dq_fp8"), ("nf4", "fp32"), ("fp4", "dq_int8")])
def test_merge_formats(codebook, fmt):
    N, K, r, s = 200, 1024, 16, 2.0
    W = _weights((N, K), 17)
    A = workloads.normal_bf16((r, K), 0.02, 18)
    B = workloads.normal_bf16((N, r), 0.02, 19)
    st = nf4.quantize_weight(W.numpy(), codebook=codebook, scale_format=fmt)
    W_hat = nf4.dequantize_weight(st, "fp32").astype(np.float64)
    out = gpu_quantize(W, CB[codebook], SF[fmt])
    Y = torch.empty((N, K), dtype=torch.float32, device="cuda")
    binding.qlora_merge(out, A.cuda(), B.cuda(), r, s, Y, 1)
    torch.cuda.synchronize()
    ref = lora.merge(W_hat, _np(A), _np(B), s)
    bound = 4 * s * (r + 1) * 2.0 ** -24 * (np.abs(_np(B)) @ np.abs(_np(A))) + 2.0 ** -24 * np.abs(ref)
    assert np.all(np.abs(_np(Y) - ref) <= bound + 1e-38)
    B0 = torch.zeros((N, r), dtype=torch.bfloat16, device="cuda")
    binding.qlora_merge(out, A.cuda(), B0, r, s, Y, 1)
    torch.cuda.synchronize()
    assert np.array_equal(Y.cpu().numpy(), nf4.dequantize_weight(st, "fp32"))


def test_format_arguments_are_checked():
    W = workloads.normal_f32((8, 128), 0.02, 1).cuda()
    ws = torch.empty(binding.qlora_nf4_sizes(8, 128)["ws_bytes"], dtype=torch.uint8, device="cuda")
    bad = binding.NF4Weight.empty(8, 128)
    bad.codebook = 2
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_nf4_quantize_ex(W, bad, ws)
    bad = binding.NF4Weight.empty(8, 128)
    bad.scale_format = 3
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_nf4_quantize_ex(W, bad, ws)
    no_absmax = binding.NF4Weight.empty(8, 128, scale_format=binding.SCALES_FP32)
    no_absmax.absmax = None
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_nf4_quantize_ex(W, no_absmax, ws)
    mixed = [binding.NF4Weight.empty(8, 128), binding.NF4Weight.empty(8, 128, codebook=binding.CODEBOOK_FP4)]
    wsb = torch.empty(binding.qlora_nf4_quantize_batched_ws_bytes(mixed), dtype=torch.uint8, device="cuda")
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_nf4_quantize_batched_ex([W, W], mixed, wsb)
    Wh = torch.zeros(8 * 128 + 8, dtype=torch.bfloat16, device="cuda")[4:4 + 8 * 128].view(8, 128)  # 8-byte offset
    with pytest.raises(binding.QloraError, match="ALIGNMENT"):
        binding.qlora_nf4_quantize_ex(Wh, binding.NF4Weight.empty(8, 128), ws)


@pytest.mark.parametrize("codebook,fmt", FORMATS)
def test_zero_second_level_scale(codebook, fmt):
    """c2 = 0 in every chunk: an all-zero weight, and a weight whose blocks all
    share one absmax (every block scale equals the mean).  The scale codes are
    0, the decoded scale is the mean, and the state and the fp32 dequantized
    weight are bit-exact with the oracle's."""
    zero = np.zeros((8, 1024), np.float32)
    same = np.tile(np.linspace(-0.5, 0.5, 64, dtype=np.float32), (8, 16))
    for W, what in ((zero, "all zero"), (same, "one absmax")):
        st = nf4.quantize_weight(W, codebook=codebook, scale_format=fmt)
        out = gpu_quantize(torch.from_numpy(W), CB[codebook], SF[fmt])
        assert_state_equal(out, st, f"{what} {codebook}/{fmt}")
        d32 = torch.empty(W.shape, dtype=torch.float32, device="cuda")
        binding.qlora_nf4_dequantize(out, d32, 1)
        torch.cuda.synchronize()
        assert np.array_equal(f32_bits(d32.cpu().numpy()), f32_bits(nf4.dequantize_weight(st, "fp32"))), what
