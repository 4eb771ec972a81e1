"""GPU parity: merged weight W_hat + s B A (qlora_merge) against the fp64 oracle.

fp32 output: each element is checked against an error bound that follows
from the kernel's arithmetic.  The decoded weight is exact in fp32.  The
rank-r sum is a tensor-core product of bf16 operands (each product exact in
fp32) accumulated in fp32 in groups of 16; the groups' summands may be
aligned and truncated rather than rounded, so the bound allows each of the
r + 1 summands 4 units of u = 2^-24 relative to sum_j |B A|.  One more
rounding of the result: u |out|.  bf16 output: the same plus one bf16
rounding of the fp32 result (2^-8 |out|).  The requantize composition (merge in fp32,
then quantize) is compared bit-exactly with the oracle's quantizer applied to
the same fp32 merged weight.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import assert_close, assert_state_equal, bf16_to_np, gpu_quantize, require_gpu
from oracle import lora, nf4

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24
U16 = 2.0 ** -8


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


def _np(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def _run_merge(out, A, B, r, s, dtype):
    Y = torch.empty((out.rows, out.cols), dtype=torch.float32 if dtype == 1 else torch.bfloat16, device="cuda")
    binding.qlora_merge(out, A, B, r, s, Y, dtype)
    torch.cuda.synchronize()
    return Y


def _check_bound(got, W_hat, A, B, r, s, unit, what):
    """Elementwise: |got - ref| <= 4 |s| (r + 1) u sum_j |B A| + unit |ref|."""
    ref = lora.merge(W_hat, A, B, s)
    bound = 4 * abs(s) * (r + 1) * U32 * (np.abs(B) @ np.abs(A)) + unit * np.abs(ref)
    err = np.abs(got - ref)
    bad = np.argwhere(err > bound + 1e-38)
    assert bad.size == 0, f"{what}: {len(bad)} elements off, first {bad[:4].tolist()} err {err[tuple(bad[0])]:.3e}"
    assert_close(got, ref, what)


def _case(N, K, r, seed, w_std=0.02, ab_std=0.02):
    W = workloads.normal_f32((N, K), w_std, seed)
    A = workloads.normal_bf16((r, K), ab_std, seed + 1)
    B = workloads.normal_bf16((N, r), ab_std, seed + 2)
    st = nf4.quantize_weight(W.numpy())
    W_hat = nf4.dequantize_weight(st, "fp32").astype(np.float64)
    return W, A, B, st, W_hat


@pytest.mark.parametrize(
    "N,K,r,b_off",
    [
        (1024, 1024, 8, 0),   # tiny configuration shape
        (6, 192, 1, 0),       # rows not a multiple of 4, one partial thread block, rank 1
        (40, 4160, 64, 1),    # ragged K tail, rank 64, A and B off a 4-byte boundary
        (8, 64, 16, 0),       # one quantization block per row
        (37, 320, 20, 0),     # ragged rows, five stripes (one CTA partly idle), rank 20
        (200, 1024, 33, 1),   # rank 33: three 16-wide steps, the last one partial
    ],
)
def test_merge_matches_oracle(N, K, r, b_off):
    W, A, B, st, W_hat = _case(N, K, r, 500 + N + K + r)
    s = 32.0 / r
    out = gpu_quantize(W)
    Bbuf = torch.zeros(N * r + 8, dtype=torch.bfloat16, device="cuda")
    Bd = Bbuf[b_off:b_off + N * r].view(N, r)
    Bd.copy_(B.cuda())
    Abuf = torch.zeros(r * K + 8, dtype=torch.bfloat16, device="cuda")
    Ad = Abuf[b_off:b_off + r * K].view(r, K)
    Ad.copy_(A.cuda())
    An, Bn = _np(A), _np(B)
    Y32 = _run_merge(out, Ad, Bd, r, s, 1)
    _check_bound(_np(Y32), W_hat, An, Bn, r, s, U32, f"fp32 {N}x{K} r={r}")
    Y16 = _run_merge(out, Ad, Bd, r, s, 0)
    _check_bound(bf16_to_np(Y16), W_hat, An, Bn, r, s, U16 + 2 * U32, f"bf16 {N}x{K} r={r}")
    # The bf16 output is the fp32 output rounded once.
    assert torch.equal(Y32.to(torch.bfloat16), Y16)


def test_merge_with_zero_b_is_the_dequantized_weight():
    """B = 0: the merged fp32 weight equals the oracle's fp32 decode exactly."""
    W, A, _, st, W_hat = _case(64, 1024, 16, 9)
    out = gpu_quantize(W)
    B0 = torch.zeros((64, 16), dtype=torch.bfloat16, device="cuda")
    Y = _run_merge(out, A.cuda(), B0, 16, 2.0, 1).cpu().numpy()
    assert np.array_equal(Y, nf4.dequantize_weight(st, "fp32"))


def test_requantizing_the_merge():
    """Merge in fp32, requantize: bit-exact with the oracle's quantizer on the
    same fp32 weight; with B = 0 the requantized codes are the original ones,
    with a nonzero adapter some codes move."""
    N, K, r = 256, 2048, 16
    W, A, B, st, W_hat = _case(N, K, r, 31, ab_std=0.05)
    out = gpu_quantize(W)
    for Bt, what in ((torch.zeros_like(B), "B=0"), (B, "B")):
        M32 = _run_merge(out, A.cuda(), Bt.cuda(), r, 2.0, 1)
        req = gpu_quantize(M32)
        st_req = nf4.quantize_weight(M32.cpu().numpy())
        assert_state_equal(req, st_req, f"requantized merge ({what})")
        same = np.array_equal(st_req.packed, st.packed)
        assert same == (what == "B=0"), f"{what}: codes {'moved' if not same else 'kept'}"


def test_merge_full_gate_projection():
    """The 14336 x 4096 gate projection, r = 16, alpha = 32, bf16 output."""
    case = workloads.gemv_case(1)
    st = nf4.quantize_weight(case.W.numpy())
    W_hat = nf4.dequantize_weight(st, "fp32").astype(np.float64)
    out = gpu_quantize(case.W)
    Y = _run_merge(out, case.A.cuda(), case.B.cuda(), case.r, case.s, 0)
    rows = np.random.default_rng(14).choice(14336, 512, replace=False)
    An, Bn = _np(case.A), _np(case.B)
    got = bf16_to_np(Y)[rows]
    _check_bound(got, W_hat[rows], An, Bn[rows], case.r, case.s, U16 + 2 * U32, "gate bf16 rows")


def test_merge_rejects_bad_arguments():
    W, A, B, st, W_hat = _case(8, 128, 4, 3)
    out = gpu_quantize(W)
    Y = torch.empty((8, 128), dtype=torch.float32, device="cuda")
    Ad, Bd = A.cuda(), B.cuda()
    for r, dtype, scale in ((0, 1, 1.0), (65, 1, 1.0), (4, 2, 1.0), (4, 1, float("inf"))):
        with pytest.raises(binding.QloraError):
            binding.qlora_merge(out, Ad, Bd, r, scale, Y, dtype)
    Ybuf = torch.empty(8 * 128 + 4, dtype=torch.float32, device="cuda")
    with pytest.raises(binding.QloraError, match="ALIGNMENT"):
        binding.qlora_merge(out, Ad, Bd, 4, 1.0, Ybuf[2:2 + 8 * 128].view(8, 128), 1)
