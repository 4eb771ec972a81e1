"""The workspace-free quantize entry point gives the same bits as the workspace one.

Callers that cannot allocate device memory (a host that reserved all device
memory in its own pool and forbids allocation while it runs, or a C caller
without a device allocator) use qlora_nf4_quantize_noalloc, whose scratch is a
fixed array inside the library.  This file is collected last so that a run
stopping at the first failure has already run every other test; it must also
pass alone in a fresh process, where its first call sets the scratch up.
"""

import numpy as np
import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding, workloads
from gpu_helpers import f32_bits, gpu_quantize, require_gpu

pytestmark = pytest.mark.gpu


def _same_state(a: binding.NF4Weight, b: binding.NF4Weight, what: str):
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed), f"{what}: packed codes differ"
    assert torch.equal(a.qscale, b.qscale), f"{what}: scale codes differ"
    assert np.array_equal(f32_bits(a.c2.cpu().numpy()), f32_bits(b.c2.cpu().numpy())), f"{what}: c2 differs"
    assert np.array_equal(f32_bits(a.mu.cpu().numpy()), f32_bits(b.mu.cpu().numpy())), f"{what}: mu differs"


def test_noalloc_matches_workspace_entry_point_on_consecutive_calls():
    require_gpu()
    shapes = [(1024, 1024), (257, 4160), (1024, 1024)]
    for i, shape in enumerate(shapes):
        W = workloads.normal_f32(shape, 0.02, 900 + i)
        W[0, :64] = 0.0
        want = gpu_quantize(W)  # the workspace entry point
        got = binding.NF4Weight.empty(*shape)
        if i == 1:
            d_status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
            binding.qlora_nf4_quantize_noalloc(W.cuda(), got, d_status=d_status)
            torch.cuda.synchronize()
            assert d_status.item() == 0
        else:
            binding.qlora_nf4_quantize_noalloc(W.cuda(), got)
        _same_state(got, want, f"call {i} {shape}")


def test_noalloc_rejects_tensors_beyond_its_scratch():
    require_gpu()
    small = binding.NF4Weight.empty(8, 64)
    big = binding.QloraNf4WeightC(1 << 14, (1 << 12) + 64, small.packed.data_ptr(), small.qscale.data_ptr(),
                                  small.c2.data_ptr(), small.mu.data_ptr())
    import ctypes

    W = torch.zeros(64, dtype=torch.float32, device="cuda")
    st = binding.lib().qlora_nf4_quantize_noalloc(W.data_ptr(), ctypes.byref(big), None,
                                                  torch.cuda.current_stream().cuda_stream)
    assert st == 7  # QLORA_ERR_UNSUPPORTED, nothing enqueued


def _same_any_format(a: binding.NF4Weight, b: binding.NF4Weight, what: str):
    if a.scale_format != binding.SCALES_FP32:
        _same_state(a, b, what)
        return
    torch.cuda.synchronize()
    assert torch.equal(a.packed, b.packed), f"{what}: packed codes differ"
    assert np.array_equal(f32_bits(a.absmax.cpu().numpy()), f32_bits(b.absmax.cpu().numpy())), f"{what}: absmax differs"


def test_noalloc_fills_its_scratch_exactly():
    """16384 x 4096 = 2^26 weights, the largest tensor the static scratch takes
    (4096 chunks of 16384 weights): the same bits as the workspace entry point."""
    require_gpu()
    shape = (16384, 4096)
    W = workloads.normal_f32(shape, 0.02, 931)
    W[-1, -64:] = 0.0  # the last block of the last chunk: the zero-block rule at the scratch's end
    want = gpu_quantize(W)
    got = binding.NF4Weight.empty(*shape)
    d_status = torch.full((1,), -1, dtype=torch.int32, device="cuda")
    binding.qlora_nf4_quantize_noalloc(W.cuda(), got, d_status=d_status)
    torch.cuda.synchronize()
    assert d_status.item() == 0
    _same_state(got, want, "2^26 weights")


def test_noalloc_refuses_one_block_past_its_scratch():
    """2^26 + 64 weights (one block more than the scratch holds) is refused on
    the host before anything is enqueued; 2^26 exactly is accepted by the
    same check."""
    require_gpu()
    import ctypes

    small = binding.NF4Weight.empty(8, 64)
    W = torch.zeros(64, dtype=torch.float32, device="cuda")
    over = binding.QloraNf4WeightC((1 << 20) + 1, 64, small.packed.data_ptr(), small.qscale.data_ptr(),
                                   small.c2.data_ptr(), small.mu.data_ptr())
    st = binding.lib().qlora_nf4_quantize_noalloc(W.data_ptr(), ctypes.byref(over), None,
                                                  torch.cuda.current_stream().cuda_stream)
    assert st == 7  # QLORA_ERR_UNSUPPORTED


@pytest.mark.parametrize("codebook,scale_format", [
    (binding.CODEBOOK_FP4, binding.SCALES_DQ_INT8),
    (binding.CODEBOOK_NF4, binding.SCALES_DQ_FP8),
    (binding.CODEBOOK_FP4, binding.SCALES_FP32),
])
def test_noalloc_other_formats(codebook, scale_format):
    """FP4 codes, E4M3 scale codes and fp32 scales through the workspace-free
    entry point: the same bits as the workspace entry point."""
    require_gpu()
    shape = (513, 4160)
    W = workloads.normal_f32(shape, 0.02, 940 + 3 * codebook + scale_format)
    W[3, 64:128] = 0.0
    want = gpu_quantize(W, codebook, scale_format)
    got = binding.NF4Weight.empty(*shape, codebook=codebook, scale_format=scale_format)
    binding.qlora_nf4_quantize_noalloc(W.cuda(), got)
    _same_any_format(got, want, f"codebook {codebook} scales {scale_format}")
