"""Every fp32 value in [-1, 1] through the GPU quantizer's FP4 decision.

The FP4 codebook has its own decision table (floor cells with a guard cell
at each end, positions mapped to sign-magnitude codes).  As for NF4, all
2,130,706,434 fp32 values x in [-1, 1] are packed 63 to a block whose 64th
weight is 1.0 (block absmax 1, normalised value x).  The expected code is
order[#{j : x >= T_j}], with T the oracle's FP4 thresholds and order the
codes by increasing level (the higher code first on the +0 / -0 tie, whose
duplicated threshold skips -0).  tests/test_oracle_formats.py pins this map
to the argmin definition on the CPU.  The file runs last: it is the longest
GPU check.
"""

import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding
from gpu_helpers import require_gpu
from oracle import nf4

pytestmark = pytest.mark.gpu

SLICE = 1 << 28  # fp32 patterns per pass (about 1 GB of weights)


def _fp4_order():
    levels = nf4.CODEBOOKS["fp4"]
    return sorted(range(16), key=lambda c: (float(levels[c]), -c))


def test_every_fp32_in_unit_interval_fp4():
    require_gpu()
    T = torch.from_numpy(nf4.decision_thresholds("fp4")).cuda()
    order = torch.tensor(_fp4_order(), dtype=torch.int64, device="cuda")
    plus_one = int(_fp4_order()[-1])  # the code of +1.0
    total = 0
    for lo_all, hi_all in ((0x00000000, 0x3F800001), (0x80000000, 0xBF800001)):
        for lo in range(lo_all, hi_all, SLICE):
            hi = min(lo + SLICE, hi_all)
            n = hi - lo
            rows = (n + 62) // 63
            bits = torch.arange(lo, lo + rows * 63, dtype=torch.int64, device="cuda")
            bits = torch.where(bits < hi, bits, torch.full_like(bits, lo))
            vals = (bits & 0xFFFFFFFF).to(torch.int32).view(torch.float32).view(rows, 63)
            W = torch.empty((rows, 64), dtype=torch.float32, device="cuda")
            W[:, :63] = vals
            W[:, 63] = 1.0
            out = binding.NF4Weight.empty(rows, 64, codebook=binding.CODEBOOK_FP4)
            ws = torch.empty(binding.qlora_nf4_sizes(rows, 64)["ws_bytes"], dtype=torch.uint8, device="cuda")
            binding.qlora_nf4_quantize_ex(W, out, ws)
            packed = out.packed.view(rows, 32)
            codes = torch.stack([packed & 15, packed >> 4], dim=2).view(rows, 64)
            got = codes[:, :63].reshape(-1)[:n].to(torch.int64)
            expect = order[torch.bucketize(vals.reshape(-1)[:n], T, right=True)]
            bad = torch.nonzero(got != expect)
            assert bad.numel() == 0, f"{bad.numel()} codes differ, first at pattern {lo + int(bad[0, 0]):#010x}"
            assert torch.all(codes[:, 63] == plus_one)
            total += n
            del W, out, ws, bits, vals, packed, codes, got, expect
            torch.cuda.empty_cache()
    assert total == 2_130_706_434
