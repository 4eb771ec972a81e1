"""GPU parity: LoRA linear forward / backward against the fp64 oracle.

Tolerance (bf16 inputs, fp32 accumulation): max |err| <= 1e-2 max|ref| and
relative Frobenius error <= 5e-3.  The oracle works on its own bf16
dequantized weight, which the quantize tests show is bit-identical to the
library's; the remaining differences are accumulation order and the bf16
rounding of outputs and of the rank-r intermediates.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, bf16_to_np, gpu_quantize, require_gpu, workspace
from oracle import lora, nf4

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _w_hat(W: torch.Tensor):
    st = nf4.quantize_weight(W.cpu().numpy())
    return st, nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _run_fwd(out, X, A, B, r, s, ws, want_u=True):
    M, N = X.shape[0], out.rows
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, r), dtype=torch.float32, device="cuda") if want_u else None
    binding.qlora_linear_fwd(out, X, A, B, r, s, Y, U, ws)
    return Y, U


def _run_bwd(out, X, dY, A, B, r, s, ws, dX_init=None, U=None):
    M, K, N = X.shape[0], out.cols, out.rows
    dX = dX_init.clone() if dX_init is not None else torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    binding.qlora_linear_bwd(out, X, dY, A, B, r, s, dX, 1 if dX_init is not None else 0, dA, dB, ws, U=U)
    return dX, dA, dB


def test_tiny_config_forward_backward():
    c = workloads.tiny_case()
    st, Wh = _w_hat(c.W)
    out = gpu_quantize(c.W)
    X, A, B, dY = (t.cuda() for t in (c.X, c.A, c.B, c.dY))
    ws = workspace(16, 1024, 1024, c.r)
    Y, U = _run_fwd(out, X, A, B, c.r, c.s, ws)
    dX, dA, dB = _run_bwd(out, X, dY, A, B, c.r, c.s, ws, U=U)
    assert binding.qlora_workspace_status(ws) == 0
    Y_ref, U_ref = lora.lora_forward(_np(c.X), Wh, _np(c.A), _np(c.B), c.s)
    dX_ref, dA_ref, dB_ref, _ = lora.lora_backward(_np(c.X), _np(c.dY), Wh, _np(c.A), _np(c.B), c.s)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(_np(U), U_ref, "U")
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert_close(_np(dA), dA_ref, "dA")
    assert_close(_np(dB), dB_ref, "dB")


def test_zero_b_gives_exactly_zero_dA():
    c = workloads.tiny_case()
    st, Wh = _w_hat(c.W)
    out = gpu_quantize(c.W)
    B0 = torch.zeros_like(c.B)
    X, A, B, dY = (t.cuda() for t in (c.X, c.A, B0, c.dY))
    ws = workspace(16, 1024, 1024, c.r)
    Y, _ = _run_fwd(out, X, A, B, c.r, c.s, ws, want_u=False)
    dX, dA, dB = _run_bwd(out, X, dY, A, B, c.r, c.s, ws)
    torch.cuda.synchronize()
    assert torch.count_nonzero(dA.view(torch.int32)).item() == 0, "dA must be all-zero bits when B = 0"
    assert dB.abs().sum().item() > 0 and dX.float().abs().sum().item() > 0
    assert_close(bf16_to_np(Y), _np(c.X) @ Wh.T, "Y with B = 0")


@pytest.mark.parametrize("M,N,K,r", [(200, 136, 320, 8), (129, 264, 192, 24), (300, 512, 1024, 64), (17, 4096, 640, 16)])
def test_tensor_core_path_ragged(M, N, K, r):
    seed = M + N + K + r
    W = workloads.normal_f32((N, K), 0.02, seed)
    A = workloads.normal_bf16((r, K), 0.02, seed + 1)
    B = workloads.normal_bf16((N, r), 0.02, seed + 2)
    X = workloads.normal_bf16((M, K), 1.0, seed + 3)
    dY = workloads.normal_bf16((M, N), 1.0, seed + 4)
    s = 2.0
    st, Wh = _w_hat(W)
    out = gpu_quantize(W)
    ws = workspace(M, N, K, r)
    Xd, Ad, Bd, dYd = (t.cuda() for t in (X, A, B, dY))
    Y, U = _run_fwd(out, Xd, Ad, Bd, r, s, ws)
    dX, dA, dB = _run_bwd(out, Xd, dYd, Ad, Bd, r, s, ws)
    dX0 = workloads.normal_bf16((M, K), 1.0, seed + 5).cuda()
    dXa, dAu, dBu = _run_bwd(out, Xd, dYd, Ad, Bd, r, s, ws, dX_init=dX0, U=U)
    assert binding.qlora_workspace_status(ws) == 0
    Y_ref, U_ref = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    dX_ref, dA_ref, dB_ref, _ = lora.lora_backward(_np(X), _np(dY), Wh, _np(A), _np(B), s)
    assert_close(bf16_to_np(Y), Y_ref, "Y")
    assert_close(_np(U), U_ref, "U")
    assert_close(bf16_to_np(dX), dX_ref, "dX")
    assert_close(bf16_to_np(dXa), dX_ref + _np(dX0), "dX accumulate")
    assert_close(_np(dA), dA_ref, "dA")
    assert_close(_np(dB), dB_ref, "dB")
    assert_close(_np(dAu), dA_ref, "dA (saved U)")
    assert_close(_np(dBu), dB_ref, "dB (saved U)")


@pytest.fixture(scope="module")
def gate7b():
    case = workloads.gemv_case(16)
    st, Wh = _w_hat(case.W)
    return case, gpu_quantize(case.W), Wh


@pytest.mark.parametrize("M", [1, 4, 16])
def test_decode_gemv_full_gate_projection(gate7b, M):
    """Decode-shaped forward at the full 14336 x 4096 gate projection."""
    case, out, Wh = gate7b
    X = workloads.normal_bf16((M, 4096), 1.0, 3000 + M)
    ws = workspace(M, 14336, 4096, case.r)
    Y, U = _run_fwd(out, X.cuda(), case.A.cuda(), case.B.cuda(), case.r, case.s, ws)
    assert binding.qlora_workspace_status(ws) == 0
    Y_ref, U_ref = lora.lora_forward(_np(X), Wh, _np(case.A), _np(case.B), case.s)
    assert_close(bf16_to_np(Y), Y_ref, f"Y M={M}")
    assert_close(_np(U), U_ref, f"U M={M}")


def test_decode_gemv_and_tensor_core_path_agree(gate7b):
    """M = 16 (GEMV) and M = 17 (tensor cores) on the same weight and rows."""
    case, out, Wh = gate7b
    X = workloads.normal_bf16((17, 4096), 1.0, 77)
    ws = workspace(17, 14336, 4096, case.r)
    Y17, _ = _run_fwd(out, X.cuda(), case.A.cuda(), case.B.cuda(), case.r, case.s, ws, want_u=False)
    Y16, _ = _run_fwd(out, X[:16].cuda(), case.A.cuda(), case.B.cuda(), case.r, case.s, ws, want_u=False)
    Y_ref, _ = lora.lora_forward(_np(X), Wh, _np(case.A), _np(case.B), case.s)
    assert_close(bf16_to_np(Y17), Y_ref, "Y M=17")
    assert_close(bf16_to_np(Y16), Y_ref[:16], "Y M=16")


@pytest.mark.parametrize(
    "M,N,K,r,b_off",
    [
        (3, 40, 192, 8, 0),        # K below one unit, most warps idle
        (1, 8, 64, 1, 0),          # one block, rank 1
        (9, 64, 1024, 64, 1),      # B not 16-byte aligned: padded copy
        (5, 136, 4160, 24, 1),     # two chunks, the last one block wide
        (16, 4096, 14336, 16, 0),  # 7B down projection: four chunks
    ],
)
def test_decode_gemv_shapes(M, N, K, r, b_off):
    """Decode path over ragged K (partial and multiple 4096-wide chunks), rank
    1 .. 64 and a B whose rows start off a 16-byte boundary."""
    seed = 7 * M + N + K + r
    W = workloads.normal_f32((N, K), 0.02, seed)
    A = workloads.normal_bf16((r, K), 0.02, seed + 1)
    B = workloads.normal_bf16((N, r), 0.02, seed + 2)
    X = workloads.normal_bf16((M, K), 1.0, seed + 3)
    s = 2.0
    st, Wh = _w_hat(W)
    out = gpu_quantize(W)
    Bbuf = torch.zeros(N * r + 8, dtype=torch.bfloat16, device="cuda")
    Bd = Bbuf[b_off:b_off + N * r].view(N, r)
    Bd.copy_(B.cuda())
    ws = workspace(M, N, K, r)
    Y, U = _run_fwd(out, X.cuda(), A.cuda(), Bd, r, s, ws)
    assert binding.qlora_workspace_status(ws) == 0
    Y_ref, U_ref = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    assert_close(bf16_to_np(Y), Y_ref, f"Y {M}x{N}x{K} r={r}")
    assert_close(_np(U), U_ref, f"U {M}x{N}x{K} r={r}")


@pytest.mark.parametrize("t", range(7))
def test_layer7b_projection_full_size(t):
    """Training-shaped 7B projection at 8192 tokens, r = 16, alpha = 32:
    64 sampled rows of Y and dX, and all of dA and dB, against the oracle."""
    case = workloads.layer7b_case(t, m=8192)
    st, Wh = _w_hat(case.W)
    out = gpu_quantize(case.W)
    M, N, K = 8192, case.proj.n, case.proj.k
    ws = workspace(M, N, K, case.r)
    X, A, B, dY = (x.cuda() for x in (case.X, case.A, case.B, case.dY))
    Y, U = _run_fwd(out, X, A, B, case.r, case.s, ws)
    dX, dA, dB = _run_bwd(out, X, dY, A, B, case.r, case.s, ws, U=U)
    assert binding.qlora_workspace_status(ws) == 0
    rows = np.random.default_rng(100 + t).choice(M, 64, replace=False)
    Xn, An, Bn, dYn = _np(case.X), _np(case.A), _np(case.B), _np(case.dY)
    assert_close(bf16_to_np(Y)[rows], lora.lora_forward_rows(rows, Xn, Wh, An, Bn, case.s), "Y rows")
    assert_close(bf16_to_np(dX)[rows], lora.lora_backward_rows(rows, dYn, Wh, An, Bn, case.s), "dX rows")
    dA_ref, dB_ref = lora.lora_adapter_grads(Xn, dYn, An, Bn, case.s)
    assert_close(_np(dA), dA_ref, "dA")
    assert_close(_np(dB), dB_ref, "dB")
