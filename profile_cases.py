"""Bounded single-kernel cases for profiler captures (a harness beside
``bench.py``, not part of the library package).

``python profile_cases.py --case gemm --reps 3`` sets up one realistic case (inputs larger than L2, a few hundred MB on the
device at most), runs the library call ``reps`` times and exits; a profiler
pointed at it with a kernel filter and a launch count captures the kernel of
interest.  The cases use the 7B gate projection (14336 x 4096) at 8192
tokens, the decode shape (16 tokens, or ``--decode-tokens``) for the GEMV, and the bf16 merged
weight (r = 16) for the merge.  ``--path dense`` runs the tensor-core calls on
the dense-weight ablation path instead of the default fused one.
"""

from __future__ import annotations

import argparse
import os
import sys

import torch

sys.path.insert(0, os.path.dirname(os.path.abspath(__file__)))

from bit_nf4_quantized_blk_b200 import binding, workloads  # noqa: E402

CASES = ("gemm", "gemm_bwd", "quantize", "dequant", "gemv", "side", "merge")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--case", choices=CASES, required=True)
    ap.add_argument("--reps", type=int, default=3)
    ap.add_argument("--tokens", type=int, default=8192)
    ap.add_argument("--decode-tokens", type=int, default=16, help="tokens of the gemv case (1..16)")
    ap.add_argument("--path", choices=("fused", "dense"), default="fused")
    args = ap.parse_args()
    torch.cuda.set_device(0)
    binding.qlora_linear_set_weight_path(
        binding.WEIGHT_PATH_DENSE if args.path == "dense" else binding.WEIGHT_PATH_FUSED)
    M = args.decode_tokens if args.case == "gemv" else (16 if args.case == "merge" else args.tokens)
    case = workloads.linear_case(workloads.GATE7B, M, 16, 32.0, 4, 0, 4, device="cuda", with_dy=args.case not in ("gemv", "merge"))
    out = binding.NF4Weight.empty(case.proj.n, case.proj.k)
    qws = torch.empty(binding.qlora_nf4_sizes(case.proj.n, case.proj.k)["ws_bytes"], dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize(case.W, out, qws)
    ws = torch.empty(binding.qlora_linear_ws_bytes(M, case.proj.n, case.proj.k, 16), dtype=torch.uint8, device="cuda")
    binding.qlora_workspace_reset(ws)
    N, K = case.proj.n, case.proj.k
    Y = torch.empty((M, N), dtype=torch.bfloat16, device="cuda")
    for _ in range(args.reps):
        if args.case in ("gemm", "gemv"):
            binding.qlora_linear_fwd(out, case.X, case.A, case.B, 16, case.s, Y, None, ws)
        elif args.case == "gemm_bwd":
            dX = torch.empty((M, K), dtype=torch.bfloat16, device="cuda")
            binding.qlora_linear_bwd(out, case.X, case.dY, case.A, case.B, 16, case.s, dX, 0, None, None, ws)
        elif args.case == "quantize":
            binding.qlora_nf4_quantize(case.W, out, qws)
        elif args.case == "dequant":
            dense = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
            binding.qlora_nf4_dequantize(out, dense, 0, 0)
        elif args.case == "merge":
            merged = torch.empty((N, K), dtype=torch.bfloat16, device="cuda")
            binding.qlora_merge(out, case.A, case.B, 16, case.s, merged, 0)
        elif args.case == "side":
            dA = torch.empty((16, K), dtype=torch.float32, device="cuda")
            dB = torch.empty((N, 16), dtype=torch.float32, device="cuda")
            binding.qlora_linear_bwd(out, case.X, case.dY, case.A, case.B, 16, case.s, None, 0, dA, dB, ws)
    torch.cuda.synchronize()
    assert binding.qlora_workspace_status(ws) == 0
    print(f"profile case {args.case}: ok")


if __name__ == "__main__":
    main()
