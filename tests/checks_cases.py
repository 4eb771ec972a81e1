"""Small odd-shaped calls through every entry point of one build of the
library, saved to a file: ``python tests/checks_cases.py LIB OUT``.

test_gpu_checks_build.py runs it as a child process once with the default
library and once with the debug library (QLORA_CHECKS: index and alignment
tests compiled in) and compares the two files.  Shapes: ragged row tiles
(N = 136), K of one block, of three blocks and past one 4096-wide chunk,
ranks 1, 8 and 24, and tokens 1, 3, 16 (decode GEMV), 17 and 33 (tensor
cores), with every codebook and scale format.
"""

from __future__ import annotations

import os
import sys

import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

from bit_nf4_quantized_blk_b200 import binding, workloads  # noqa: E402


def _quantize(W, codebook, fmt):
    rows, cols = W.shape
    out = binding.NF4Weight.empty(rows, cols, codebook=codebook, scale_format=fmt)
    ws = torch.empty(binding.qlora_nf4_sizes(rows, cols)["ws_bytes"], dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize_ex(W, out, ws)
    return out


def run(out_path: str) -> None:
    res = {}
    probe = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    binding.qlora_selftest_checks(probe)
    res["checks_probe"] = probe.cpu()
    formats = [(cb, sf) for cb in (binding.CODEBOOK_NF4, binding.CODEBOOK_FP4)
               for sf in (binding.SCALES_DQ_INT8, binding.SCALES_DQ_FP8, binding.SCALES_FP32)]
    for cb, sf in formats:
        W = workloads.normal_f32((136, 192), 0.02, 11 + cb * 3 + sf).cuda()
        out = _quantize(W, cb, sf)
        for name in ("packed", "qscale", "c2", "mu", "absmax"):
            t = getattr(out, name, None)
            if t is not None:
                res[f"q{cb}{sf}/{name}"] = t.cpu()
        dense = torch.empty((136, 192), dtype=torch.bfloat16, device="cuda")
        binding.qlora_nf4_dequantize(out, dense, 0, 0)
        res[f"q{cb}{sf}/dequant"] = dense.cpu()

    for N, K, r in ((136, 64, 1), (136, 192, 8), (40, 4160, 24)):
        W = workloads.normal_f32((N, K), 0.02, N + K + r).cuda()
        out = _quantize(W, binding.CODEBOOK_NF4, binding.SCALES_DQ_INT8)
        A = workloads.normal_bf16((r, K), 0.02, r + 1).cuda()
        B = workloads.normal_bf16((N, r), 0.02, r + 2).cuda()
        for M in (1, 3, 16, 17, 33):
            X = workloads.normal_bf16((M, K), 1.0, M + 3).cuda()
            dY = workloads.normal_bf16((M, N), 1.0, M + 4).cuda()
            ws = torch.empty(binding.qlora_linear_ws_bytes(M, N, K, r), dtype=torch.uint8, device="cuda")
            binding.qlora_workspace_reset(ws)
            Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
            U = torch.empty((M, r), dtype=torch.float32, device="cuda")
            binding.qlora_linear_fwd(out, X, A, B, r, 2.0, Y, U, ws)
            dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
            dA = torch.empty((r, K), dtype=torch.float32, device="cuda")
            dB = torch.empty((N, r), dtype=torch.float32, device="cuda")
            binding.qlora_linear_bwd(out, X, dY, A, B, r, 2.0, dX, 0, dA, dB, ws, U=U)
            key = f"lin{N}x{K}r{r}M{M}"
            res[key + "/status"] = torch.tensor(binding.qlora_workspace_status(ws))
            for name, t in (("Y", Y), ("U", U), ("dX", dX), ("dA", dA), ("dB", dB)):
                res[f"{key}/{name}"] = t.cpu()
        merged = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
        binding.qlora_merge(out, A, B, r, 2.0, merged, 0)
        res[f"merge{N}x{K}r{r}"] = merged.cpu()
    torch.cuda.synchronize()
    torch.save(res, out_path)


if __name__ == "__main__":
    binding.LIB_PATH = os.path.abspath(sys.argv[1])
    torch.cuda.set_device(0)
    run(sys.argv[2])
