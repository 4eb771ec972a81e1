"""The C ABI library loads and exports every entry point its header declares.

CPU-only: no call here reaches a GPU.  Host-side size arithmetic and argument
checks return before anything is enqueued, so they run without a device.
"""

import ctypes
import os
import re

import pytest

from bit_nf4_quantized_blk_b200 import binding

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    names = []
    inc = os.path.join(ROOT, "include")
    for fname in sorted(os.listdir(inc)):
        if not fname.endswith(".h"):
            continue
        text = open(os.path.join(inc, fname)).read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        names += re.findall(r"^\s*(?:const\s+)?[a-z_0-9]+\s*\*?\s*(qlora_[a-z_0-9]+)\s*\(", text, flags=re.M)
    return sorted(set(names))


@pytest.fixture(scope="module")
def lib():
    from bit_nf4_quantized_blk_b200 import build

    build.build()
    return binding.lib()


def test_header_declares_the_four_method_calls():
    names = _declared_functions()
    for n in ("qlora_nf4_quantize", "qlora_nf4_dequantize", "qlora_linear_fwd", "qlora_linear_bwd"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    names = _declared_functions()
    assert len(names) >= 12
    for n in names:
        assert hasattr(lib, n), n
    assert sorted(names) == sorted(binding.EXPORTED)


def test_checks_library_exports_the_same_symbols():
    """The debug library (QLORA_CHECKS: index and alignment tests compiled in)
    is built beside the default one and has the same C ABI."""
    from bit_nf4_quantized_blk_b200 import build

    path = build.build(checks=True)
    assert path.endswith("libqlora_nf4_checks.so") and os.path.exists(path)
    L = ctypes.CDLL(path)
    for n in _declared_functions():
        assert hasattr(L, n), n


def test_status_strings(lib):
    assert binding.qlora_status_string(0) == "ok"
    assert "workspace" in binding.qlora_status_string(4)
    assert "check" in binding.qlora_status_string(8)
    assert binding.STATUS_NAMES[8] == "QLORA_ERR_CHECK"
    assert binding.qlora_status_string(99) == "unknown status"


def test_ring_selftest_arguments_checked_on_the_host(lib):
    """Out-of-range self-test arguments are refused before any launch."""
    f = lib.qlora_selftest_mbarrier_ring
    buf = ctypes.c_void_p(256)  # never dereferenced: every call below is refused first
    for args in ((0, 1, 16, 1000), (9, 1, 16, 1000), (2, 5, 16, 1000), (2, -1, 16, 1000), (2, 1, 0, 1000),
                 (2, 1, (1 << 24) + 1, 1000), (2, 1, 16, 0), (2, 1, 16, 1000001)):
        assert f(*args, buf, None) == 1, args
    assert f(2, 1, 16, 1000, None, None) == 1
    assert lib.qlora_selftest_checks(None, None) == 1


def test_sizes(lib):
    s = binding.qlora_nf4_sizes(1024, 1024)
    assert s["packed_bytes"] == 1024 * 1024 // 2
    assert s["n_blocks"] == 1024 * 1024 // 64
    assert s["n_chunks"] == 64
    assert s["ws_bytes"] >= 256 + 64 * 256 * 4
    s = binding.qlora_nf4_sizes(3, 192)  # 9 blocks: one partial chunk
    assert s["n_blocks"] == 9 and s["n_chunks"] == 1
    for rows, cols in ((0, 64), (4, 0), (4, 96), (-1, 64)):
        with pytest.raises(binding.QloraError) as e:
            binding.qlora_nf4_sizes(rows, cols)
        assert e.value.status == 1


def test_linear_ws_bytes(lib):
    assert binding.qlora_linear_weight_path() == binding.WEIGHT_PATH_FUSED  # the default
    # the fused path holds no dense copy of the weight; the dense-weight
    # ablation path adds one of N x K bf16 for the tensor-core calls (M > 16)
    fused = binding.qlora_linear_ws_bytes(8192, 14336, 4096, 16)
    assert 0 < fused < 14336 * 4096 * 2  # smaller than a bf16 copy of the weight alone
    with binding.weight_path(binding.WEIGHT_PATH_DENSE):
        # the dense arm holds the N x K bf16 copy (it needs no decoded-scale array, N x K / 64 fp32)
        assert binding.qlora_linear_ws_bytes(8192, 14336, 4096, 16) >= fused + 14336 * 4096 * 2 - 14336 * 64 * 4
        decode_dense = binding.qlora_linear_ws_bytes(16, 1024, 1024, 8)
    assert binding.qlora_linear_weight_path() == binding.WEIGHT_PATH_FUSED
    # M <= 16: the forward is the GEMV, but the backward's GEMM still reads the copy on the dense path
    assert decode_dense >= binding.qlora_linear_ws_bytes(16, 1024, 1024, 8) + 1024 * 1024 * 2 - 1024 * 16 * 4
    assert binding.qlora_linear_ws_bytes(0, 1024, 1024, 8) == 0
    assert binding.qlora_linear_ws_bytes(16, 1024, 1000, 8) == 0
    assert binding.qlora_linear_ws_bytes(16, 1024, 1024, 65) == 0
    assert binding.qlora_linear_ws_bytes(16, 1020, 1024, 8) == 0  # N not a multiple of 8
    assert binding.qlora_linear_ws_bytes(2**25, 8, 64, 8) > 0  # the largest M the calls take
    assert binding.qlora_linear_ws_bytes(2**25 + 1, 8, 64, 8) == 0
    assert binding.qlora_linear_ws_bytes(16, 2**33, 64, 8) == 0  # N beyond 32-bit indices
    assert binding.qlora_linear_ws_bytes(16, 8, 2**31, 8) == 0  # K likewise


def test_weight_path_selector(lib):
    L = binding.lib()
    assert L.qlora_linear_set_weight_path(2) == 1  # QLORA_ERR_INVALID_ARG
    assert L.qlora_linear_set_weight_path(-1) == 1
    assert L.qlora_linear_weight_path() == binding.WEIGHT_PATH_FUSED
    assert L.qlora_linear_set_weight_path(binding.WEIGHT_PATH_DENSE) == 0
    assert L.qlora_linear_weight_path() == binding.WEIGHT_PATH_DENSE
    assert L.qlora_linear_set_weight_path(binding.WEIGHT_PATH_FUSED) == 0
    assert L.qlora_linear_weight_path() == binding.WEIGHT_PATH_FUSED


def test_linear_size_limits_refused_on_the_host(lib):
    """A weight whose row count passes the storage checks but exceeds the
    linear kernels' 32-bit indices is refused (7 = QLORA_ERR_UNSUPPORTED)
    before the workspace or the device is looked at."""
    W = binding.QloraNf4WeightC(2**33, 64, 16, 16, 16, 16)
    assert lib.qlora_linear_fwd(ctypes.byref(W), 16, 4, 16, 16, 8, 1.0, 16, None, 256, 1 << 30, None) == 7
    assert lib.qlora_linear_bwd(ctypes.byref(W), 16, 16, 4, 16, 16, 8, 1.0, None, 16, 0, None, None, 256,
                                1 << 30, None) == 7
    W8 = binding.QloraNf4WeightC(8, 64, 16, 16, 16, 16)
    assert lib.qlora_linear_fwd(ctypes.byref(W8), 16, 2**25 + 1, 16, 16, 8, 1.0, 16, None, 256, 1 << 30,
                                None) == 7


def test_argument_checks_run_before_any_launch(lib):
    W = binding.QloraNf4WeightC(64, 64, 0, 0, 0, 0)  # null device pointers
    st = lib.qlora_nf4_quantize(None, ctypes.byref(W), None, 0, None, None)
    assert st == 1  # INVALID_ARG: nothing enqueued
    W2 = binding.QloraNf4WeightC(64, 64, 16, 16, 16, 16)
    st = lib.qlora_nf4_quantize(32, ctypes.byref(W2), None, 0, None, None)
    assert st == 4  # WORKSPACE
    st = lib.qlora_nf4_quantize(32, ctypes.byref(W2), 256, 1 << 20, None, None)
    assert st in (5, 7)  # no device here: CUDA error / unsupported, never a launch
    W3 = binding.QloraNf4WeightC(64, 64, 17, 16, 16, 16)
    assert lib.qlora_nf4_quantize(32, ctypes.byref(W3), 256, 1 << 20, None, None) == 2  # ALIGNMENT
    W4 = binding.QloraNf4WeightC(64, 100, 16, 16, 16, 16)
    assert lib.qlora_nf4_dequantize(ctypes.byref(W4), 16, 0, 0, None) == 1
    assert lib.qlora_nf4_dequantize(ctypes.byref(W2), 16, 2, 0, None) == 1  # bad dtype
    assert lib.qlora_linear_fwd(ctypes.byref(W2), 16, 4, 16, 16, 0, 1.0, 16, None, 256, 1 << 30, None) == 1  # r = 0
    assert lib.qlora_linear_fwd(ctypes.byref(W2), 16, 4, 16, 16, 8, 1.0, 16, None, 256, 16, None) == 4  # small ws
    assert lib.qlora_linear_bwd(ctypes.byref(W2), 16, 16, 4, 16, 16, 8, 1.0, None, None, 2, None, None, 256,
                                1 << 30, None) == 1  # accumulate must be 0 or 1


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "_lib", None)
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError):
        binding.lib()


def _enum_values(name):
    text = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    body = re.search(r"typedef enum " + name + r"\s*\{(.*?)\}", text, flags=re.S).group(1)
    return {k: int(v) for k, v in re.findall(r"(QLORA_[A-Z0-9_]+)\s*=\s*(\d+)", body)}


def test_format_constants_match_the_header():
    assert _enum_values("qlora_codebook") == {"QLORA_CODEBOOK_NF4": binding.CODEBOOK_NF4,
                                              "QLORA_CODEBOOK_FP4": binding.CODEBOOK_FP4}
    assert _enum_values("qlora_scale_format") == {"QLORA_SCALES_DQ_INT8": binding.SCALES_DQ_INT8,
                                                  "QLORA_SCALES_DQ_FP8": binding.SCALES_DQ_FP8,
                                                  "QLORA_SCALES_FP32": binding.SCALES_FP32}
    assert _enum_values("qlora_input_dtype") == {"QLORA_INPUT_FP32": binding.INPUT_FP32,
                                                 "QLORA_INPUT_BF16": binding.INPUT_BF16,
                                                 "QLORA_INPUT_FP16": binding.INPUT_FP16}


def test_weight_descriptor_layout_matches_the_header():
    """The ctypes descriptor has the header's fields in the header's order."""
    text = open(os.path.join(ROOT, "include", "qlora_nf4.h")).read()
    body = re.search(r"typedef struct qlora_nf4_weight\s*\{(.*?)\}", text, flags=re.S).group(1)
    fields = re.findall(r"\*?\s*([a-z_0-9]+);", body)
    assert fields == [f for f, _ in binding.QloraNf4WeightC._fields_]
    assert ctypes.sizeof(binding.QloraNf4WeightC) == 64


def test_format_arguments_rejected_on_the_host(lib):
    """Invalid codebook / scale format / missing absmax are refused before any
    device work (the checks run on the host): status 1 = QLORA_ERR_INVALID_ARG."""
    st = binding.QloraNf4WeightC(8, 128, 16, 16, 16, 16, 2, 0, None)
    out = ctypes.c_void_p(16)
    assert lib.qlora_nf4_dequantize(ctypes.byref(st), out, 0, 0, None) == 1
    st = binding.QloraNf4WeightC(8, 128, 16, 16, 16, 16, 0, 3, None)
    assert lib.qlora_nf4_dequantize(ctypes.byref(st), out, 0, 0, None) == 1
    st = binding.QloraNf4WeightC(8, 128, 16, None, None, None, 0, binding.SCALES_FP32, None)
    assert lib.qlora_nf4_dequantize(ctypes.byref(st), out, 0, 0, None) == 1
