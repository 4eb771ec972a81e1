"""Thin ctypes binding of ``libqlora_nf4.so`` (the C ABI in include/qlora_nf4.h).

Argument marshalling only: every function takes torch tensors (device memory
owned by the caller), passes their data pointers and the current CUDA stream
to the C entry point of the same name, and raises :class:`QloraError` on a
non-OK status.  No step of the computation runs here.  Loading fails loudly
if the shared library has not been built.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libqlora_nf4.so")

QLORA_OK = 0
STATUS_NAMES = {
    0: "QLORA_OK",
    1: "QLORA_ERR_INVALID_ARG",
    2: "QLORA_ERR_ALIGNMENT",
    3: "QLORA_ERR_NONFINITE",
    4: "QLORA_ERR_WORKSPACE",
    5: "QLORA_ERR_CUDA",
    6: "QLORA_ERR_TIMEOUT",
    7: "QLORA_ERR_UNSUPPORTED",
}

EXPORTED = [
    "qlora_status_string",
    "qlora_nf4_sizes",
    "qlora_nf4_quantize",
    "qlora_nf4_quantize_batched_ws_bytes",
    "qlora_nf4_quantize_batched",
    "qlora_nf4_quantize_noalloc",
    "qlora_nf4_quantize_ex",
    "qlora_nf4_quantize_batched_ex",
    "qlora_nf4_dequantize",
    "qlora_nf4_dequantize_batched",
    "qlora_merge",
    "qlora_workspace_reset",
    "qlora_workspace_status",
    "qlora_linear_ws_bytes",
    "qlora_linear_fwd",
    "qlora_linear_bwd",
    "qlora_timing_enable",
    "qlora_timing_read",
]


class QloraError(RuntimeError):
    def __init__(self, fn: str, status: int):
        self.status = status
        super().__init__(f"{fn} failed: {STATUS_NAMES.get(status, status)}")


# qlora_codebook, qlora_scale_format and qlora_input_dtype of the header.
CODEBOOK_NF4, CODEBOOK_FP4 = 0, 1
SCALES_DQ_INT8, SCALES_DQ_FP8, SCALES_FP32 = 0, 1, 2
INPUT_FP32, INPUT_BF16, INPUT_FP16 = 0, 1, 2
_INPUT_OF_DTYPE = {torch.float32: INPUT_FP32, torch.bfloat16: INPUT_BF16, torch.float16: INPUT_FP16}


class QloraNf4WeightC(ctypes.Structure):
    _fields_ = [
        ("rows", ctypes.c_int64),
        ("cols", ctypes.c_int64),
        ("packed", ctypes.c_void_p),
        ("qscale", ctypes.c_void_p),
        ("c2", ctypes.c_void_p),
        ("mu", ctypes.c_void_p),
        ("codebook", ctypes.c_int32),
        ("scale_format", ctypes.c_int32),
        ("absmax", ctypes.c_void_p),
    ]


_lib = None


def lib() -> ctypes.CDLL:
    """The loaded library; raises if it has not been built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m bit_nf4_quantized_blk_b200.build`"
        )
    L = ctypes.CDLL(LIB_PATH)
    P = ctypes.c_void_p
    i32, i64, sz, f32 = ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
    W = ctypes.POINTER(QloraNf4WeightC)
    sig = {
        "qlora_status_string": (ctypes.c_char_p, [i32]),
        "qlora_nf4_sizes": (i32, [i64, i64, ctypes.POINTER(sz), ctypes.POINTER(sz), ctypes.POINTER(sz),
                                  ctypes.POINTER(sz)]),
        "qlora_nf4_quantize": (i32, [P, W, P, sz, P, P]),
        "qlora_nf4_quantize_batched_ws_bytes": (sz, [W, i32]),
        "qlora_nf4_quantize_batched": (i32, [ctypes.POINTER(P), W, i32, P, sz, P, P]),
        "qlora_nf4_quantize_noalloc": (i32, [P, W, P, P]),
        "qlora_nf4_quantize_ex": (i32, [P, i32, W, P, sz, P, P]),
        "qlora_nf4_quantize_batched_ex": (i32, [ctypes.POINTER(P), i32, W, i32, P, sz, P, P]),
        "qlora_nf4_dequantize": (i32, [W, P, i32, i32, P]),
        "qlora_nf4_dequantize_batched": (i32, [W, ctypes.POINTER(P), i32, i32, P]),
        "qlora_merge": (i32, [W, P, P, i32, f32, P, i32, P]),
        "qlora_workspace_reset": (i32, [P, sz, P]),
        "qlora_workspace_status": (i32, [P, sz, P]),
        "qlora_linear_ws_bytes": (sz, [i64, i64, i64, i32]),
        "qlora_linear_fwd": (i32, [W, P, i64, P, P, i32, f32, P, P, P, sz, P]),
        "qlora_linear_bwd": (i32, [W, P, P, i64, P, P, i32, f32, P, P, i32, P, P, P, sz, P]),
        "qlora_timing_enable": (i32, [i32]),
        "qlora_timing_read": (i32, [ctypes.c_char_p, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(i64)]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(L, name)
        fn.restype = res
        fn.argtypes = args
    _lib = L
    return L


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _stream(stream) -> int | None:
    if stream is None:
        return torch.cuda.current_stream().cuda_stream
    return stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)


def _check(fn: str, status: int) -> None:
    if status != QLORA_OK:
        raise QloraError(fn, status)


@dataclass
class NF4Weight:
    """Device buffers of one quantized tensor (caller-owned torch tensors)."""

    rows: int
    cols: int
    packed: torch.Tensor  # uint8 [rows*cols/2]
    qscale: torch.Tensor | None  # int8 [rows*cols/64] (int8 or E4M3 codes); None for fp32 scales
    c2: torch.Tensor | None  # fp32 [n_chunks]; None for fp32 scales
    mu: torch.Tensor | None  # fp32 [1]; None for fp32 scales
    codebook: int = CODEBOOK_NF4
    scale_format: int = SCALES_DQ_INT8
    absmax: torch.Tensor | None = None  # fp32 [rows*cols/64] for fp32 scales

    @classmethod
    def empty(cls, rows: int, cols: int, device="cuda", codebook: int = CODEBOOK_NF4,
              scale_format: int = SCALES_DQ_INT8) -> "NF4Weight":
        s = qlora_nf4_sizes(rows, cols)
        packed = torch.empty(s["packed_bytes"], dtype=torch.uint8, device=device)
        if scale_format == SCALES_FP32:
            return cls(rows, cols, packed, None, None, None, codebook, scale_format,
                       torch.empty(s["n_blocks"], dtype=torch.float32, device=device))
        return cls(
            rows,
            cols,
            packed,
            torch.empty(s["n_blocks"], dtype=torch.int8, device=device),
            torch.empty(s["n_chunks"], dtype=torch.float32, device=device),
            torch.empty(1, dtype=torch.float32, device=device),
            codebook,
            scale_format,
        )

    def c_struct(self) -> QloraNf4WeightC:
        return QloraNf4WeightC(self.rows, self.cols, self.packed.data_ptr(), _ptr(self.qscale), _ptr(self.c2),
                               _ptr(self.mu), self.codebook, self.scale_format, _ptr(self.absmax))


def qlora_status_string(status: int) -> str:
    return lib().qlora_status_string(status).decode()


def qlora_nf4_sizes(rows: int, cols: int) -> dict:
    vals = [ctypes.c_size_t() for _ in range(4)]
    _check("qlora_nf4_sizes", lib().qlora_nf4_sizes(rows, cols, *[ctypes.byref(v) for v in vals]))
    keys = ("packed_bytes", "n_blocks", "n_chunks", "ws_bytes")
    return {k: v.value for k, v in zip(keys, vals)}


def qlora_nf4_quantize(W: torch.Tensor, out: NF4Weight, ws: torch.Tensor, d_status=None, stream=None) -> None:
    st = out.c_struct()
    _check("qlora_nf4_quantize", lib().qlora_nf4_quantize(W.data_ptr(), ctypes.byref(st), ws.data_ptr(),
                                                          ws.numel() * ws.element_size(), _ptr(d_status),
                                                          _stream(stream)))


def qlora_nf4_quantize_ex(W: torch.Tensor, out: NF4Weight, ws: torch.Tensor, d_status=None, stream=None) -> None:
    """Quantize an fp32, bf16 or fp16 tensor (the input dtype follows W.dtype)."""
    st = out.c_struct()
    _check("qlora_nf4_quantize_ex",
           lib().qlora_nf4_quantize_ex(W.data_ptr(), _INPUT_OF_DTYPE[W.dtype], ctypes.byref(st), ws.data_ptr(),
                                       ws.numel() * ws.element_size(), _ptr(d_status), _stream(stream)))


def qlora_nf4_quantize_batched_ex(Ws, outs, ws: torch.Tensor, d_status=None, stream=None) -> None:
    dtypes = {w.dtype for w in Ws}
    if len(dtypes) != 1:
        raise ValueError("one input dtype per call")
    arr = _weight_array(outs)
    ptrs = (ctypes.c_void_p * len(Ws))(*[w.data_ptr() for w in Ws])
    _check("qlora_nf4_quantize_batched_ex",
           lib().qlora_nf4_quantize_batched_ex(ptrs, _INPUT_OF_DTYPE[dtypes.pop()], arr, len(outs), ws.data_ptr(),
                                               ws.numel() * ws.element_size(), _ptr(d_status), _stream(stream)))


def _weight_array(ws):
    arr = (QloraNf4WeightC * len(ws))()
    for i, w in enumerate(ws):
        arr[i] = w.c_struct()
    return arr


def qlora_nf4_quantize_batched_ws_bytes(outs) -> int:
    arr = _weight_array(outs)
    return int(lib().qlora_nf4_quantize_batched_ws_bytes(arr, len(outs)))


def qlora_nf4_quantize_batched(Ws, outs, ws: torch.Tensor, d_status=None, stream=None) -> None:
    arr = _weight_array(outs)
    ptrs = (ctypes.c_void_p * len(Ws))(*[w.data_ptr() for w in Ws])
    _check("qlora_nf4_quantize_batched",
           lib().qlora_nf4_quantize_batched(ptrs, arr, len(outs), ws.data_ptr(), ws.numel() * ws.element_size(),
                                            _ptr(d_status), _stream(stream)))


def qlora_nf4_quantize_noalloc(W: torch.Tensor, out: NF4Weight, d_status=None, stream=None) -> None:
    """Quantize without a workspace (library-internal scratch; tensors up to 2^26 weights)."""
    st = out.c_struct()
    _check("qlora_nf4_quantize_noalloc",
           lib().qlora_nf4_quantize_noalloc(W.data_ptr(), ctypes.byref(st), _ptr(d_status), _stream(stream)))


def qlora_nf4_dequantize(w: NF4Weight, out: torch.Tensor, out_dtype: int = 0, transpose: int = 0, stream=None) -> None:
    st = w.c_struct()
    _check("qlora_nf4_dequantize",
           lib().qlora_nf4_dequantize(ctypes.byref(st), out.data_ptr(), out_dtype, transpose, _stream(stream)))


def qlora_nf4_dequantize_batched(weights, outs, out_dtype: int = 0, stream=None) -> None:
    arr = _weight_array(weights)
    ptrs = (ctypes.c_void_p * len(outs))(*[o.data_ptr() for o in outs])
    _check("qlora_nf4_dequantize_batched",
           lib().qlora_nf4_dequantize_batched(arr, ptrs, len(weights), out_dtype, _stream(stream)))


def qlora_merge(w: NF4Weight, A, B, r: int, scale: float, out, out_dtype: int = 0, stream=None) -> None:
    st = w.c_struct()
    _check("qlora_merge",
           lib().qlora_merge(ctypes.byref(st), A.data_ptr(), B.data_ptr(), r, float(scale), out.data_ptr(),
                             out_dtype, _stream(stream)))


def qlora_workspace_reset(ws: torch.Tensor, stream=None) -> None:
    _check("qlora_workspace_reset", lib().qlora_workspace_reset(ws.data_ptr(), ws.numel(), _stream(stream)))


def qlora_workspace_status(ws: torch.Tensor, stream=None) -> int:
    return int(lib().qlora_workspace_status(ws.data_ptr(), ws.numel(), _stream(stream)))


def qlora_linear_ws_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_linear_ws_bytes(M, N, K, r))


def qlora_linear_fwd(w: NF4Weight, X, A, B, r: int, scale: float, Y, U_out, ws, stream=None) -> None:
    st = w.c_struct()
    _check("qlora_linear_fwd",
           lib().qlora_linear_fwd(ctypes.byref(st), X.data_ptr(), X.shape[0], A.data_ptr(), B.data_ptr(), r,
                                  float(scale), Y.data_ptr(), _ptr(U_out), ws.data_ptr(), ws.numel(),
                                  _stream(stream)))


def qlora_linear_bwd(w: NF4Weight, X, dY, A, B, r: int, scale: float, dX, accumulate: int, dA, dB, ws,
                     U=None, stream=None) -> None:
    st = w.c_struct()
    _check("qlora_linear_bwd",
           lib().qlora_linear_bwd(ctypes.byref(st), X.data_ptr(), dY.data_ptr(), X.shape[0], A.data_ptr(),
                                  B.data_ptr(), r, float(scale), _ptr(U), _ptr(dX), int(accumulate), _ptr(dA),
                                  _ptr(dB), ws.data_ptr(), ws.numel(), _stream(stream)))


def qlora_timing_enable(enable: bool) -> None:
    _check("qlora_timing_enable", lib().qlora_timing_enable(1 if enable else 0))


def qlora_timing_read(family: str) -> tuple[float, int]:
    """(summed device milliseconds, launches) of a kernel family since enabling."""
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    _check("qlora_timing_read", lib().qlora_timing_read(family.encode(), ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value
