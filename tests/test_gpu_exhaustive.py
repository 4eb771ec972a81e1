"""Every fp32 value in [-1, 1] through the GPU quantizer's nearest-level decision.

All 2,130,706,434 fp32 values x in [-1, 1] (both zeros included) are packed 63
to a 64-weight block whose 64th weight is 1.0, so the block absmax is 1 and the
kernel's normalised value is x itself.  Each code must equal the oracle's:
code(x) = #{j : x >= T_j} with the oracle's thresholds, which the CPU tests pin
to the argmin definition (the choice between neighbouring levels flips once).
"""

import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding
from gpu_helpers import require_gpu
from oracle import nf4

pytestmark = pytest.mark.gpu

SLICE = 1 << 28  # fp32 patterns per pass (about 1 GB of weights)


def _codes_of_patterns(lo: int, hi: int, thresholds: torch.Tensor):
    """GPU codes and expected codes of the fp32 bit patterns [lo, hi)."""
    n = hi - lo
    rows = (n + 62) // 63
    bits = torch.arange(lo, lo + rows * 63, dtype=torch.int64, device="cuda")
    bits = torch.where(bits < hi, bits, torch.full_like(bits, lo))  # pad the tail with a valid value
    vals = (bits & 0xFFFFFFFF).to(torch.int32).view(torch.float32).view(rows, 63)
    W = torch.empty((rows, 64), dtype=torch.float32, device="cuda")
    W[:, :63] = vals
    W[:, 63] = 1.0
    out = binding.NF4Weight.empty(rows, 64)
    ws = torch.empty(binding.qlora_nf4_sizes(rows, 64)["ws_bytes"], dtype=torch.uint8, device="cuda")
    binding.qlora_nf4_quantize(W, out, ws)
    packed = out.packed.view(rows, 32)
    codes = torch.stack([packed & 15, packed >> 4], dim=2).view(rows, 64)[:, :63].reshape(-1)[:n]
    expect = torch.bucketize(vals.reshape(-1)[:n], thresholds, right=True)
    last = torch.stack([packed[:, 31] >> 4]).reshape(-1)
    return codes.to(torch.int64), expect, last


def test_every_fp32_in_unit_interval():
    require_gpu()
    T = torch.from_numpy(nf4.decision_thresholds()).cuda()
    total = 0
    for lo_all, hi_all in ((0x00000000, 0x3F800001), (0x80000000, 0xBF800001)):
        for lo in range(lo_all, hi_all, SLICE):
            hi = min(lo + SLICE, hi_all)
            codes, expect, last = _codes_of_patterns(lo, hi, T)
            bad = torch.nonzero(codes != expect)
            assert bad.numel() == 0, f"{bad.numel()} codes differ, first at pattern {lo + int(bad[0, 0]):#010x}"
            assert torch.all(last == 15)  # the 1.0 of every block
            total += hi - lo
            del codes, expect, last
            torch.cuda.empty_cache()
    assert total == 2_130_706_434
