"""GPU: the tensor-core linear calls with the 4-bit weight decoded inside the
GEMM (the default path) against the dense-weight ablation path and the oracle.

Both paths decode the same bf16 weight values and accumulate each output tile
in the same order, so Y and dX must agree bit for bit; every case is also
checked against the fp64 oracle within the stated tolerance.  The shapes cover
ragged token counts, weight rows that end inside a 256-row tile (forward) or a
64-row reduction stage (backward), K that is not a multiple of 256, ranks 1 to
64, every stored format, and accumulation into dX.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, bf16_to_np, gpu_quantize, require_gpu, workspace
from oracle import lora, nf4

pytestmark = pytest.mark.gpu

FORMATS = {
    "nf4_int8": (binding.CODEBOOK_NF4, binding.SCALES_DQ_INT8, "nf4", "dq_int8"),
    "nf4_fp8": (binding.CODEBOOK_NF4, binding.SCALES_DQ_FP8, "nf4", "dq_fp8"),
    "nf4_fp32": (binding.CODEBOOK_NF4, binding.SCALES_FP32, "nf4", "fp32"),
    "fp4_int8": (binding.CODEBOOK_FP4, binding.SCALES_DQ_INT8, "fp4", "dq_int8"),
}


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()
    yield
    binding.qlora_linear_set_weight_path(binding.WEIGHT_PATH_FUSED)


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _both_paths(out, X, dY, A, B, r, s, dX0):
    """(Y, dX, dX accumulated, dA, dB) on the fused and on the dense path."""
    M, N, K = X.shape[0], out.rows, out.cols
    res = {}
    for path in (binding.WEIGHT_PATH_FUSED, binding.WEIGHT_PATH_DENSE):
        with binding.weight_path(path):
            ws = workspace(M, N, K, r)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            U = torch.empty((M, r), dtype=torch.float32, device="cuda")
            binding.qlora_linear_fwd(out, X, A, B, r, s, Y, U, ws)
            dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
            dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
            dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
            binding.qlora_linear_bwd(out, X, dY, A, B, r, s, dX, 0, dA, dB, ws, U=U)
            dXa = dX0.clone()
            binding.qlora_linear_bwd(out, X, dY, A, B, r, s, dXa, 1, None, None, ws, U=U)
            assert binding.qlora_workspace_status(ws) == 0
            res[path] = (Y, dX, dXa, dA, dB)
    return res[binding.WEIGHT_PATH_FUSED], res[binding.WEIGHT_PATH_DENSE]


def _bits_equal(a, b, what):
    ai, bi = a.view(torch.int16) if a.dtype == torch.bfloat16 else a.view(torch.int32), \
        b.view(torch.int16) if b.dtype == torch.bfloat16 else b.view(torch.int32)
    diff = (ai != bi).nonzero()
    assert diff.numel() == 0, f"{what}: fused and dense paths differ at {diff[:4].tolist()}"


@pytest.mark.parametrize(
    "M,N,K,r",
    [
        (16, 1024, 1024, 8),     # decode-sized M: GEMV forward, tensor-core backward on both paths
        (17, 8, 64, 1),          # one weight row, one block per row, rank 1
        (200, 136, 320, 8),      # N ends inside a tile and a reduction stage; K % 256 != 0
        (129, 264, 192, 24),
        (300, 512, 1024, 64),    # largest rank: four K = 16 rank steps
        (513, 1032, 704, 16),    # three token tiles, the last holding one row
        (256, 4096, 640, 5),
    ],
)
@pytest.mark.parametrize("fmt", list(FORMATS))
def test_fused_matches_dense_bit_for_bit(M, N, K, r, fmt):
    codebook, scales, cb_name, sc_name = FORMATS[fmt]
    seed = 3 * M + N + K + r + codebook * 7 + scales * 11
    W = workloads.normal_f32((N, K), 0.02, seed)
    A = workloads.normal_bf16((r, K), 0.02, seed + 1).cuda()
    B = workloads.normal_bf16((N, r), 0.02, seed + 2).cuda()
    X = workloads.normal_bf16((M, K), 1.0, seed + 3).cuda()
    dY = workloads.normal_bf16((M, N), 1.0, seed + 4).cuda()
    dX0 = workloads.normal_bf16((M, K), 1.0, seed + 5).cuda()
    s = 2.0
    out = gpu_quantize(W, codebook, scales)
    fused, dense = _both_paths(out, X, dY, A, B, r, s, dX0)
    for name, f, d in zip(("Y", "dX", "dX accumulate", "dA", "dB"), fused, dense):
        _bits_equal(f, d, f"{fmt} {M}x{N}x{K} r={r} {name}")
    # and the oracle, on the oracle's own bf16 weight of the same format
    st = nf4.quantize_weight(W.numpy(), codebook=cb_name, scale_format=sc_name)
    Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
    Y_ref, _ = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    dX_ref, _, _, _ = lora.lora_backward(_np(X), _np(dY), Wh, _np(A), _np(B), s)
    assert_close(bf16_to_np(fused[0]), Y_ref, f"{fmt} Y")
    assert_close(bf16_to_np(fused[1]), dX_ref, f"{fmt} dX")
    assert_close(bf16_to_np(fused[2]), dX_ref + _np(dX0), f"{fmt} dX accumulate")


def test_fused_path_needs_no_dense_weight_workspace():
    """The fused path's workspace holds no N x K copy; the dense path's does,
    and a dense call given the fused size is refused before any launch."""
    M, N, K, r = 8192, 14336, 4096, 16
    with binding.weight_path(binding.WEIGHT_PATH_FUSED):
        fused = binding.qlora_linear_ws_bytes(M, N, K, r)
    with binding.weight_path(binding.WEIGHT_PATH_DENSE):
        dense = binding.qlora_linear_ws_bytes(M, N, K, r)
    # the dense arm adds the N x K bf16 copy and drops the fused path's
    # decoded block scales (N x K / 64 fp32)
    assert dense - fused >= N * K * 2 - N * (K // 64) * 4
    assert fused < N * K * 2  # smaller than a bf16 copy of the weight alone
    W = workloads.normal_f32((64, 128), 0.02, 5)
    out = gpu_quantize(W)
    X = torch.zeros((32, 128), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((32, 64), dtype=torch.bfloat16, device="cuda")
    ws = workspace(32, 64, 128, 8)  # fused size
    with binding.weight_path(binding.WEIGHT_PATH_DENSE):
        with pytest.raises(binding.QloraError) as ei:
            binding.qlora_linear_fwd(out, X, A, B, 8, 2.0, Y, None, ws)
    assert ei.value.status == 4  # QLORA_ERR_WORKSPACE


@pytest.mark.parametrize("t", [1, 4, 6])  # k (N = 1024), gate (14336 x 4096), down (4096 x 14336)
def test_fused_matches_dense_full_size_projection(t):
    """7B projections at 8192 tokens: the two paths agree bit for bit."""
    case = workloads.layer7b_case(t, m=8192)
    out = gpu_quantize(case.W)
    X, A, B, dY = (x.cuda() for x in (case.X, case.A, case.B, case.dY))
    dX0 = torch.zeros((8192, case.proj.k), dtype=torch.bfloat16, device="cuda")
    fused, dense = _both_paths(out, X, dY, A, B, case.r, case.s, dX0)
    for name, f, d in zip(("Y", "dX", "dX accumulate", "dA", "dB"), fused, dense):
        _bits_equal(f, d, f"projection {t} {name}")
