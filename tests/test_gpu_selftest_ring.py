"""Phase-parity self-test of the shared-memory barrier ring the pipelined
kernels use (qlora_selftest_mbarrier_ring): with 1 to 4 stages and 1 or 2
consumer warps every value arrives once and in order; with no consumer the
producer's bounded wait runs out and reports QLORA_ERR_TIMEOUT (no trap, the
device stays usable)."""

import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding
from gpu_helpers import require_gpu

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu():
    require_gpu()


@pytest.mark.parametrize("stages", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("consumers", [1, 2, 4])
def test_ring_passes_every_value_in_order(stages, consumers):
    iters = 4099  # not a multiple of any ring depth: the last pass is partial
    res = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    binding.qlora_selftest_mbarrier_ring(stages, consumers, iters, 1000000, res)
    wrong, read, status = res.tolist()
    assert status == 0
    assert wrong == 0
    assert read == iters * consumers


def test_ring_without_consumer_times_out():
    res = torch.full((3,), -1, dtype=torch.int32, device="cuda")
    binding.qlora_selftest_mbarrier_ring(1, 0, 2, 2000, res)
    wrong, read, status = res.tolist()
    assert status == 6  # QLORA_ERR_TIMEOUT
    assert wrong == 0 and read == 0
    # The context is still usable: a normal ring runs right after.
    binding.qlora_selftest_mbarrier_ring(2, 1, 64, 1000000, res)
    assert res.tolist() == [0, 64, 0]
