"""GPU: a bounded device wait that runs out.

The fused GEMM's MMA issuer is made to wait on a barrier that nothing arrives
at (qlora_linear_fwd_stall_diagnostic), with every pipeline wait limited to a
few milliseconds.  The wait runs out and the pair takes its abort path: the
status word reads QLORA_ERR_TIMEOUT, the copies already issued are waited for,
tensor memory is freed and the kernel returns.  The device and the stream stay
usable: the next ordinary call on the same stream and workspace matches the
oracle, and so does a second diagnostic followed by another ordinary call.
No fault, trap or hang is involved: the failure is a flag nobody sets.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, bf16_to_np, gpu_quantize, require_gpu, workspace
from oracle import lora, nf4

pytestmark = pytest.mark.gpu

QLORA_ERR_TIMEOUT = 6


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def test_wait_timeout_is_reported_and_the_next_call_is_correct():
    M, N, K, r = 96, 512, 1024, 8
    W = workloads.normal_f32((N, K), 0.02, 71)
    A = workloads.normal_bf16((r, K), 0.02, 72)
    B = workloads.normal_bf16((N, r), 0.02, 73)
    X = workloads.normal_bf16((M, K), 1.0, 74)
    s = 2.0
    st = nf4.quantize_weight(W.numpy())
    Wh = nf4.bf16_bits_to_f32(nf4.dequantize_weight(st, "bf16")).astype(np.float64)
    Y_ref, _ = lora.lora_forward(_np(X), Wh, _np(A), _np(B), s)
    out = gpu_quantize(W)
    Xd, Ad, Bd = X.cuda(), A.cuda(), B.cuda()
    ws = workspace(M, N, K, r)
    for round_ in range(2):
        Y = torch.full((M, N), 7.0, dtype=torch.bfloat16, device="cuda")
        binding.qlora_linear_fwd_stall_diagnostic(out, Xd, Ad, Bd, r, s, Y, ws, 2000)
        assert binding.qlora_workspace_status(ws) == QLORA_ERR_TIMEOUT, f"round {round_}: timeout not reported"
        assert binding.qlora_workspace_status(ws) == 0  # reading cleared it
        binding.qlora_linear_fwd(out, Xd, Ad, Bd, r, s, Y, None, ws)
        assert binding.qlora_workspace_status(ws) == 0
        assert_close(bf16_to_np(Y), Y_ref, f"Y after timeout round {round_}")


def test_stall_diagnostic_refuses_bad_arguments():
    W = workloads.normal_f32((64, 128), 0.02, 75)
    out = gpu_quantize(W)
    X = torch.zeros((16, 128), dtype=torch.bfloat16, device="cuda")
    A = torch.zeros((8, 128), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((64, 8), dtype=torch.bfloat16, device="cuda")
    Y = torch.empty((16, 64), dtype=torch.bfloat16, device="cuda")
    ws = workspace(32, 64, 128, 8)
    for M, limit in ((16, 2000), (32, 0), (32, 2_000_000)):  # decode-sized M; limits out of range
        with pytest.raises(binding.QloraError) as ei:
            binding.qlora_linear_fwd_stall_diagnostic(out, X[:M] if M <= 16 else torch.zeros(
                (M, 128), dtype=torch.bfloat16, device="cuda"), A, B, 8, 2.0,
                Y if M <= 16 else torch.empty((M, 64), dtype=torch.bfloat16, device="cuda"), ws, limit)
        assert ei.value.status == 1
    assert binding.qlora_workspace_status(ws) == 0
