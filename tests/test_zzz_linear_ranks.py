"""GPU parity of the tensor-core linear path at ranks and B layouts that take
the zero-padded copy of B: r not a multiple of 8 (1, 5, 12) and a B whose rows
do not start on a 16-byte boundary, plus a direct-B case on a ragged K.

Forward (Y, U), backward (dX, dA, dB), the accumulate flag and the saved-U
variant against the fp64 oracle, with the tolerance of the other linear
tests (max |err| <= 1e-2 max |ref|, relative Frobenius error <= 5e-3).
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, bf16_to_np, gpu_quantize, require_gpu, workspace
from oracle import lora, nf4

pytestmark = pytest.mark.gpu


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize(
    "M,N,K,r,b_off",
    [
        (130, 200, 256, 1, 0),    # rank 1
        (97, 136, 384, 5, 0),     # odd rank
        (256, 264, 192, 12, 0),   # rank between the 8-column steps
        (97, 128, 512, 16, 1),    # B rows off a 16-byte boundary
        (40, 64, 4160, 40, 0),    # direct B, K not a multiple of 128
    ],
)
def test_padded_b_ranks(M, N, K, r, b_off):
    require_gpu()
    seed = 3 * M + N + K + r
    W = workloads.normal_f32((N, K), 0.02, seed)
    A = workloads.normal_bf16((r, K), 0.02, seed + 1)
    B = workloads.normal_bf16((N, r), 0.02, seed + 2)
    X = workloads.normal_bf16((M, K), 1.0, seed + 3)
    dY = workloads.normal_bf16((M, N), 1.0, seed + 4)
    s = 32.0 / r
    st = nf4.quantize_weight(W.numpy())
    Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
    out = gpu_quantize(W)
    ws = workspace(M, N, K, r)
    Bbuf = torch.zeros(N * r + 8, dtype=torch.bfloat16, device="cuda")
    Bd = Bbuf[b_off:b_off + N * r].view(N, r)
    Bd.copy_(B.cuda())
    Xd, Ad, dYd = X.cuda(), A.cuda(), dY.cuda()

    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    U = torch.empty((M, r), dtype=torch.float32, device="cuda")
    binding.qlora_linear_fwd(out, Xd, Ad, Bd, r, s, Y, U, ws)
    dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
    dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
    dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
    binding.qlora_linear_bwd(out, Xd, dYd, Ad, Bd, r, s, dX, 0, dA, dB, ws)
    dX0 = workloads.normal_bf16((M, K), 1.0, seed + 5).cuda()
    dXa = dX0.clone()
    dAu = torch.empty_like(dA)
    dBu = torch.empty_like(dB)
    binding.qlora_linear_bwd(out, Xd, dYd, Ad, Bd, r, s, dXa, 1, dAu, dBu, ws, U=U)
    assert binding.qlora_workspace_status(ws) == 0

    Y_ref, U_ref = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    dX_ref, dA_ref, dB_ref, _ = lora.lora_backward(_np(X), _np(dY), Wh, _np(A), _np(B), s)
    what = f"{M}x{N}x{K} r={r} b_off={b_off}"
    assert_close(bf16_to_np(Y), Y_ref, f"Y {what}")
    assert_close(_np(U), U_ref, f"U {what}")
    assert_close(bf16_to_np(dX), dX_ref, f"dX {what}")
    assert_close(bf16_to_np(dXa), dX_ref + _np(dX0), f"dX accumulate {what}")
    assert_close(_np(dA), dA_ref, f"dA {what}")
    assert_close(_np(dB), dB_ref, f"dB {what}")
    assert_close(_np(dAu), dA_ref, f"dA saved U {what}")
    assert_close(_np(dBu), dB_ref, f"dB saved U {what}")
