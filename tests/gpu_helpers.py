"""Helpers shared by the GPU parity tests (inputs, tolerance, GPU-side calls)."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding

# Tolerance for bf16-input / fp32-accumulate outputs: max |err| <= 1e-2 max|ref|
# and relative Frobenius error <= 5e-3.
MAX_REL = 1e-2
FRO_REL = 5e-3


def require_gpu():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    cap = torch.cuda.get_device_capability()
    if cap != (10, 0):
        pytest.skip(f"needs sm_100, found {cap}")
    from bit_nf4_quantized_blk_b200 import build

    build.build()
    binding.lib()


def assert_close(got, ref, what=""):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = got - ref
    scale = np.abs(ref).max()
    max_err = np.abs(err).max()
    fro = np.linalg.norm(err) / max(np.linalg.norm(ref), 1e-300)
    assert max_err <= MAX_REL * scale, f"{what}: max|err| {max_err:.3e} > {MAX_REL} * {scale:.3e}"
    assert fro <= FRO_REL, f"{what}: relative Frobenius error {fro:.3e} > {FRO_REL}"
    return max_err / max(scale, 1e-300), fro


def bf16_to_np(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def f32_bits(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32)).view(np.uint32)


def gpu_quantize(W: torch.Tensor, codebook: int = 0, scale_format: int = 0) -> binding.NF4Weight:
    """Quantize one fp32, bf16 or fp16 tensor on the GPU through the C ABI
    (status read back)."""
    rows, cols = W.shape
    Wd = W.to("cuda").contiguous()
    out = binding.NF4Weight.empty(rows, cols, codebook=codebook, scale_format=scale_format)
    ws = torch.empty(binding.qlora_nf4_sizes(rows, cols)["ws_bytes"], dtype=torch.uint8, device="cuda")
    if Wd.dtype == torch.float32 and codebook == 0 and scale_format == 0:
        binding.qlora_nf4_quantize(Wd, out, ws)
    else:
        binding.qlora_nf4_quantize_ex(Wd, out, ws)
    return out


def assert_state_equal(out: binding.NF4Weight, st, what=""):
    """Bit-exact comparison of the GPU state with the oracle's NF4DQState
    (any codebook / scale format)."""
    torch.cuda.synchronize()
    packed = out.packed.cpu().numpy()
    assert np.array_equal(packed, st.packed), f"{what}: packed codes differ at {np.flatnonzero(packed != st.packed)[:8]}"
    if st.scale_format == "fp32":
        a = f32_bits(out.absmax.cpu().numpy())
        assert np.array_equal(a, f32_bits(st.absmax)), f"{what}: absmax differs at {np.flatnonzero(a != f32_bits(st.absmax))[:8]}"
        return
    q = out.qscale.cpu().numpy().view(np.uint8)
    sq = np.asarray(st.qscale).view(np.uint8)
    assert np.array_equal(q, sq), f"{what}: scale codes differ at {np.flatnonzero(q != sq)[:8]}"
    assert np.array_equal(f32_bits(out.c2.cpu().numpy()), f32_bits(st.c2)), f"{what}: c2 differs"
    assert f32_bits(out.mu.cpu().numpy())[0] == f32_bits([st.mu])[0], f"{what}: mu {out.mu.item()} != {st.mu}"


def workspace(M, N, K, r):
    nbytes = binding.qlora_linear_ws_bytes(M, N, K, r)
    ws = torch.empty(nbytes, dtype=torch.uint8, device="cuda")
    binding.qlora_workspace_reset(ws)
    return ws
