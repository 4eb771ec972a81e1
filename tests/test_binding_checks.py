"""The binding refuses tensors whose pointers the library could not use safely.

CPU-only.  A raw device pointer carries no device, dtype, layout or size, so
the binding checks those on the torch side before any pointer reaches the
library: a CPU tensor, a non-contiguous view, a wrong dtype or a buffer
smaller than the call's extent raises here.  Arguments the library checks
itself (ranks, enum values, alignment) are left to it, so no size is derived
from an out-of-range rank.
"""

import pytest
import torch

from bit_nf4_quantized_blk_b200 import binding


@pytest.fixture(scope="module")
def w():
    from bit_nf4_quantized_blk_b200 import build

    build.build()
    return binding.NF4Weight.empty(8, 128, device="cpu")  # sizes come from the host-only size query


@pytest.fixture
def any_device(monkeypatch):
    """Let CPU tensors pass the placement check so that the checks after it
    in argument order are reached.  Every call below still fails one check
    before the library, and the library refuses host-side on a machine
    without a GPU in any case."""
    monkeypatch.setattr(binding, "_check_placement", lambda t, name: None)


def test_cpu_tensors_are_refused(w):
    W = torch.zeros(8, 128)
    ws = torch.empty(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.qlora_nf4_quantize(W, w, ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.qlora_workspace_reset(ws)
    with pytest.raises(ValueError, match="CUDA tensor"):
        binding.qlora_nf4_dequantize(w, torch.empty(8, 128, dtype=torch.bfloat16), 0)


def test_dtype_layout_and_size(w, any_device):
    ws = torch.empty(1 << 16, dtype=torch.uint8)
    with pytest.raises(TypeError, match="W: dtype"):
        binding.qlora_nf4_quantize(torch.zeros(8, 128, dtype=torch.bfloat16), w, ws)
    with pytest.raises(ValueError, match="contiguous"):
        binding.qlora_nf4_quantize(torch.zeros(128, 8).t(), w, ws)
    with pytest.raises(ValueError, match="needs at least 1024"):
        binding.qlora_nf4_quantize(torch.zeros(8, 127), w, ws)
    with pytest.raises(TypeError, match="fp32, bf16 or fp16"):
        binding.qlora_nf4_quantize_ex(torch.zeros(8, 128, dtype=torch.float64), w, ws)
    with pytest.raises(TypeError, match="out: dtype"):
        binding.qlora_nf4_dequantize(w, torch.empty(8, 128, dtype=torch.bfloat16), 1)  # fp32 output wanted
    with pytest.raises(ValueError, match="out: 1000 elements"):
        binding.qlora_nf4_dequantize(w, torch.empty(1000, dtype=torch.float32), 1)


def test_weight_buffers_are_checked(w, any_device):
    short = binding.NF4Weight(w.rows, w.cols, w.packed[:100], w.qscale, w.c2, w.mu)
    with pytest.raises(ValueError, match="packed: 100 elements, needs at least 512"):
        binding.qlora_nf4_dequantize(short, torch.empty(8, 128, dtype=torch.float32), 1)
    wrong = binding.NF4Weight(w.rows, w.cols, w.packed, w.qscale.float(), w.c2, w.mu)
    with pytest.raises(TypeError, match="qscale: dtype"):
        binding.qlora_nf4_dequantize(wrong, torch.empty(8, 128, dtype=torch.float32), 1)


def test_batches_must_pair_inputs_and_outputs(w, any_device):
    ws = torch.empty(1 << 16, dtype=torch.uint8)
    with pytest.raises(ValueError, match="2 inputs for 1 outputs"):
        binding.qlora_nf4_quantize_batched([torch.zeros(8, 128), torch.zeros(8, 128)], [w], ws)
    with pytest.raises(ValueError, match="1 inputs for 2 outputs"):
        binding.qlora_nf4_dequantize_batched([w], [torch.empty(8, 128), torch.empty(8, 128)], 1)


def test_linear_shapes(w, any_device):
    A = torch.zeros(4, 128, dtype=torch.bfloat16)
    B = torch.zeros(8, 4, dtype=torch.bfloat16)
    ws = torch.empty(1 << 16, dtype=torch.uint8)
    Y = torch.empty(32, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError, match="2-D"):
        binding.qlora_linear_fwd(w, torch.zeros(128, dtype=torch.bfloat16), A, B, 4, 1.0, Y, None, ws)
    with pytest.raises(ValueError, match="K = 128"):
        binding.qlora_linear_fwd(w, torch.zeros(32, 64, dtype=torch.bfloat16), A, B, 4, 1.0, Y, None, ws)
    with pytest.raises(ValueError, match="Y: 8 elements, needs at least 256"):
        binding.qlora_linear_fwd(w, torch.zeros(32, 128, dtype=torch.bfloat16), A, B, 4, 1.0, Y[:1], None, ws)
    with pytest.raises(ValueError, match="A: 128 elements, needs at least 512"):
        binding.qlora_linear_fwd(w, torch.zeros(32, 128, dtype=torch.bfloat16), A[:1], B, 4, 1.0, Y, None, ws)
    with pytest.raises(TypeError, match="dA: dtype"):
        binding.qlora_linear_bwd(w, torch.zeros(32, 128, dtype=torch.bfloat16), torch.zeros(32, 8, dtype=torch.bfloat16),
                                 A, B, 4, 1.0, None, 0, torch.zeros(4, 128, dtype=torch.bfloat16), None, ws)


def test_out_of_range_arguments_are_left_to_the_library(w, any_device):
    """With r = 65 or out_dtype = 2 the binding derives no size or dtype
    requirement from them: the call reaches the library, which refuses it on
    the host (QloraError, not a binding ValueError) before any pointer is
    used."""
    A = torch.zeros(4, 128, dtype=torch.bfloat16)
    B = torch.zeros(8, 4, dtype=torch.bfloat16)
    out = torch.empty(8, 128, dtype=torch.float32)
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_merge(w, A, B, 65, 1.0, out, 1, stream=0)
    with pytest.raises(binding.QloraError, match="INVALID_ARG"):
        binding.qlora_merge(w, A, B, 4, 1.0, out, 2, stream=0)
