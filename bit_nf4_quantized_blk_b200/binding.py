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
    8: "QLORA_ERR_CHECK",
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
    "qlora_linear_set_weight_path",
    "qlora_linear_weight_path",
    "qlora_linear_fwd",
    "qlora_linear_fwd_stall_diagnostic",
    "qlora_selftest_mbarrier_ring",
    "qlora_selftest_checks",
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
WEIGHT_PATH_FUSED, WEIGHT_PATH_DENSE = 0, 1  # qlora_weight_path
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
        "qlora_linear_set_weight_path": (i32, [i32]),
        "qlora_linear_weight_path": (i32, []),
        "qlora_linear_fwd": (i32, [W, P, i64, P, P, i32, f32, P, P, P, sz, P]),
        "qlora_linear_fwd_stall_diagnostic": (i32, [W, P, i64, P, P, i32, f32, P, P, sz, i32, P]),
        "qlora_selftest_mbarrier_ring": (i32, [i32, i32, i32, i32, P, P]),
        "qlora_selftest_checks": (i32, [P, P]),
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


# dtypes accepted for "bf16" buffers: bf16 data or its 16-bit patterns.
_BF16_BITS = (torch.bfloat16, torch.int16, torch.uint16)
_F32 = (torch.float32,)
_OUT_DTYPES = {0: _BF16_BITS, 1: _F32}  # out_dtype 0 = bf16, 1 = fp32


def _dev(t, name: str, dtypes=None, need: int | None = None) -> int:
    """Device pointer of tensor argument ``name`` after the checks a raw
    pointer cannot carry: a torch.Tensor, contiguous, of one of ``dtypes``,
    with at least ``need`` elements, on the current CUDA device (the device
    the library launches on).  What the library checks itself (alignment,
    weight shapes, ranks, enum values) is left to it."""
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name}: expected a torch.Tensor, got {type(t).__name__}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if dtypes is not None and t.dtype not in dtypes:
        raise TypeError(f"{name}: dtype {t.dtype}, expected one of {', '.join(str(d) for d in dtypes)}")
    if need is not None and t.numel() < need:
        raise ValueError(f"{name}: {t.numel()} elements, needs at least {need}")
    _check_placement(t, name)
    return t.data_ptr()


def _check_placement(t: torch.Tensor, name: str) -> None:
    """The tensor lives on the current CUDA device (the one the library launches on)."""
    if t.device.type != "cuda":
        raise ValueError(f"{name}: must be a CUDA tensor, got one on {t.device}")
    cur = torch.cuda.current_device()
    if t.device.index != cur:
        raise ValueError(f"{name}: on {t.device}, but the library runs on the current device cuda:{cur}")


def _dev_opt(t, name: str, dtypes=None, need: int | None = None) -> int | None:
    return None if t is None else _dev(t, name, dtypes, need)


def _ws(ws, name: str = "ws") -> tuple[int, int]:
    """(pointer, size in bytes) of a workspace tensor of any dtype."""
    return _dev(ws, name), ws.numel() * ws.element_size()


def _rank_ok(r: int) -> bool:
    return 1 <= r <= 64


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

    @property
    def numel(self) -> int | None:
        """rows * cols, or None when the shape is one the library refuses."""
        ok = self.rows >= 1 and self.cols >= 64 and self.cols % 64 == 0
        return self.rows * self.cols if ok else None

    def c_struct(self) -> QloraNf4WeightC:
        n = self.numel
        blocks = None if n is None else n // 64
        chunks = None if n is None else (blocks + 255) // 256
        return QloraNf4WeightC(
            self.rows,
            self.cols,
            _dev(self.packed, "packed", (torch.uint8,), None if n is None else n // 2),
            _dev_opt(self.qscale, "qscale", (torch.int8, torch.uint8), blocks),
            _dev_opt(self.c2, "c2", _F32, chunks),
            _dev_opt(self.mu, "mu", _F32, None if n is None else 1),
            self.codebook,
            self.scale_format,
            _dev_opt(self.absmax, "absmax", _F32, blocks),
        )


def _weight_array(ws):
    arr = (QloraNf4WeightC * len(ws))()
    for i, w in enumerate(ws):
        arr[i] = w.c_struct()
    return arr


def _same_length(a, b, what: str) -> None:
    if len(a) != len(b):
        raise ValueError(f"{what}: {len(a)} inputs for {len(b)} outputs")


def qlora_status_string(status: int) -> str:
    return lib().qlora_status_string(status).decode()


def qlora_nf4_sizes(rows: int, cols: int) -> dict:
    vals = [ctypes.c_size_t() for _ in range(4)]
    _check("qlora_nf4_sizes", lib().qlora_nf4_sizes(rows, cols, *[ctypes.byref(v) for v in vals]))
    keys = ("packed_bytes", "n_blocks", "n_chunks", "ws_bytes")
    return {k: v.value for k, v in zip(keys, vals)}


def qlora_nf4_quantize(W: torch.Tensor, out: NF4Weight, ws: torch.Tensor, d_status=None, stream=None) -> None:
    st = out.c_struct()
    wp = _dev(W, "W", _F32, out.numel)
    wsp, wsb = _ws(ws)
    dsp = _dev_opt(d_status, "d_status", (torch.int32,), 1)
    _check("qlora_nf4_quantize", lib().qlora_nf4_quantize(wp, ctypes.byref(st), wsp, wsb, dsp, _stream(stream)))


def _input_code(W: torch.Tensor, name: str) -> int:
    if not isinstance(W, torch.Tensor) or W.dtype not in _INPUT_OF_DTYPE:
        raise TypeError(f"{name}: expected an fp32, bf16 or fp16 torch.Tensor")
    return _INPUT_OF_DTYPE[W.dtype]


def qlora_nf4_quantize_ex(W: torch.Tensor, out: NF4Weight, ws: torch.Tensor, d_status=None, stream=None) -> None:
    """Quantize an fp32, bf16 or fp16 tensor (the input dtype follows W.dtype)."""
    code = _input_code(W, "W")
    st = out.c_struct()
    wp = _dev(W, "W", None, out.numel)
    wsp, wsb = _ws(ws)
    dsp = _dev_opt(d_status, "d_status", (torch.int32,), 1)
    _check("qlora_nf4_quantize_ex",
           lib().qlora_nf4_quantize_ex(wp, code, ctypes.byref(st), wsp, wsb, dsp, _stream(stream)))


def qlora_nf4_quantize_batched_ex(Ws, outs, ws: torch.Tensor, d_status=None, stream=None) -> None:
    _same_length(Ws, outs, "qlora_nf4_quantize_batched_ex")
    codes = {_input_code(w, f"Ws[{i}]") for i, w in enumerate(Ws)}
    if len(codes) > 1:
        raise ValueError("one input dtype per call")
    arr = _weight_array(outs)
    ptrs = (ctypes.c_void_p * len(Ws))(*[_dev(w, f"Ws[{i}]", None, o.numel) for i, (w, o) in enumerate(zip(Ws, outs))])
    wsp, wsb = _ws(ws)
    dsp = _dev_opt(d_status, "d_status", (torch.int32,), 1)
    code = codes.pop() if codes else INPUT_FP32
    _check("qlora_nf4_quantize_batched_ex",
           lib().qlora_nf4_quantize_batched_ex(ptrs, code, arr, len(outs), wsp, wsb, dsp, _stream(stream)))


def qlora_nf4_quantize_batched_ws_bytes(outs) -> int:
    arr = _weight_array(outs)
    return int(lib().qlora_nf4_quantize_batched_ws_bytes(arr, len(outs)))


def qlora_nf4_quantize_batched(Ws, outs, ws: torch.Tensor, d_status=None, stream=None) -> None:
    _same_length(Ws, outs, "qlora_nf4_quantize_batched")
    arr = _weight_array(outs)
    ptrs = (ctypes.c_void_p * len(Ws))(*[_dev(w, f"Ws[{i}]", _F32, o.numel) for i, (w, o) in enumerate(zip(Ws, outs))])
    wsp, wsb = _ws(ws)
    dsp = _dev_opt(d_status, "d_status", (torch.int32,), 1)
    _check("qlora_nf4_quantize_batched",
           lib().qlora_nf4_quantize_batched(ptrs, arr, len(outs), wsp, wsb, dsp, _stream(stream)))


def qlora_nf4_quantize_noalloc(W: torch.Tensor, out: NF4Weight, d_status=None, stream=None) -> None:
    """Quantize without a workspace (library-internal scratch; tensors up to 2^26 weights)."""
    st = out.c_struct()
    wp = _dev(W, "W", _F32, out.numel)
    dsp = _dev_opt(d_status, "d_status", (torch.int32,), 1)
    _check("qlora_nf4_quantize_noalloc", lib().qlora_nf4_quantize_noalloc(wp, ctypes.byref(st), dsp, _stream(stream)))


def qlora_nf4_dequantize(w: NF4Weight, out: torch.Tensor, out_dtype: int = 0, transpose: int = 0, stream=None) -> None:
    st = w.c_struct()
    op = _dev(out, "out", _OUT_DTYPES.get(out_dtype), w.numel)
    _check("qlora_nf4_dequantize", lib().qlora_nf4_dequantize(ctypes.byref(st), op, out_dtype, transpose,
                                                              _stream(stream)))


def qlora_nf4_dequantize_batched(weights, outs, out_dtype: int = 0, stream=None) -> None:
    _same_length(weights, outs, "qlora_nf4_dequantize_batched")
    arr = _weight_array(weights)
    dt = _OUT_DTYPES.get(out_dtype)
    ptrs = (ctypes.c_void_p * len(outs))(*[_dev(o, f"outs[{i}]", dt, w.numel)
                                           for i, (w, o) in enumerate(zip(weights, outs))])
    _check("qlora_nf4_dequantize_batched",
           lib().qlora_nf4_dequantize_batched(arr, ptrs, len(weights), out_dtype, _stream(stream)))


def qlora_merge(w: NF4Weight, A, B, r: int, scale: float, out, out_dtype: int = 0, stream=None) -> None:
    st = w.c_struct()
    sized = w.numel is not None and _rank_ok(r)
    ap = _dev(A, "A", _BF16_BITS, r * w.cols if sized else None)
    bp = _dev(B, "B", _BF16_BITS, w.rows * r if sized else None)
    op = _dev(out, "out", _OUT_DTYPES.get(out_dtype), w.numel)
    _check("qlora_merge", lib().qlora_merge(ctypes.byref(st), ap, bp, r, float(scale), op, out_dtype, _stream(stream)))


def qlora_workspace_reset(ws: torch.Tensor, stream=None) -> None:
    wsp, wsb = _ws(ws)
    _check("qlora_workspace_reset", lib().qlora_workspace_reset(wsp, wsb, _stream(stream)))


def qlora_workspace_status(ws: torch.Tensor, stream=None) -> int:
    wsp, wsb = _ws(ws)
    return int(lib().qlora_workspace_status(wsp, wsb, _stream(stream)))


def qlora_linear_ws_bytes(M: int, N: int, K: int, r: int) -> int:
    return int(lib().qlora_linear_ws_bytes(M, N, K, r))


def qlora_linear_set_weight_path(path: int) -> None:
    _check("qlora_linear_set_weight_path", lib().qlora_linear_set_weight_path(int(path)))


def qlora_linear_weight_path() -> int:
    return int(lib().qlora_linear_weight_path())


class weight_path:
    """Context manager: run the enclosed linear calls on `path`
    (WEIGHT_PATH_FUSED or WEIGHT_PATH_DENSE), restoring the previous path."""

    def __init__(self, path: int):
        self.path = path
        self.prev = None

    def __enter__(self):
        self.prev = qlora_linear_weight_path()
        qlora_linear_set_weight_path(self.path)
        return self

    def __exit__(self, *exc):
        qlora_linear_set_weight_path(self.prev)
        return False


def _tokens(X, name: str, w: NF4Weight) -> int:
    """M of a [M, K] activation, checking its second dimension against the weight's K."""
    if not isinstance(X, torch.Tensor) or X.dim() != 2:
        raise ValueError(f"{name}: expected a 2-D [M, K] tensor")
    if w.numel is not None and X.shape[1] != w.cols:
        raise ValueError(f"{name}: {X.shape[1]} columns, the weight has K = {w.cols}")
    return X.shape[0]


def qlora_linear_fwd(w: NF4Weight, X, A, B, r: int, scale: float, Y, U_out, ws, stream=None) -> None:
    st = w.c_struct()
    M = _tokens(X, "X", w)
    sized = w.numel is not None and _rank_ok(r)
    N, K = w.rows, w.cols
    xp = _dev(X, "X", _BF16_BITS)
    ap = _dev(A, "A", _BF16_BITS, r * K if sized else None)
    bp = _dev(B, "B", _BF16_BITS, N * r if sized else None)
    yp = _dev(Y, "Y", _BF16_BITS, M * N if w.numel is not None else None)
    up = _dev_opt(U_out, "U_out", _F32, M * r if sized else None)
    wsp, wsb = _ws(ws)
    _check("qlora_linear_fwd",
           lib().qlora_linear_fwd(ctypes.byref(st), xp, M, ap, bp, r, float(scale), yp, up, wsp, wsb, _stream(stream)))


def qlora_linear_fwd_stall_diagnostic(w: NF4Weight, X, A, B, r: int, scale: float, Y, ws, wait_limit_us: int,
                                      stream=None) -> None:
    """Diagnostic: the tensor-core forward with its GEMM made to time out
    (see the header); read the outcome with qlora_workspace_status."""
    st = w.c_struct()
    M = _tokens(X, "X", w)
    sized = w.numel is not None and _rank_ok(r)
    N, K = w.rows, w.cols
    xp = _dev(X, "X", _BF16_BITS)
    ap = _dev(A, "A", _BF16_BITS, r * K if sized else None)
    bp = _dev(B, "B", _BF16_BITS, N * r if sized else None)
    yp = _dev(Y, "Y", _BF16_BITS, M * N if w.numel is not None else None)
    wsp, wsb = _ws(ws)
    _check("qlora_linear_fwd_stall_diagnostic",
           lib().qlora_linear_fwd_stall_diagnostic(ctypes.byref(st), xp, M, ap, bp, r, float(scale), yp, wsp, wsb,
                                                   int(wait_limit_us), _stream(stream)))


def qlora_selftest_mbarrier_ring(stages: int, consumers: int, iters: int, wait_limit_us: int, result,
                                 stream=None) -> None:
    """Diagnostic: the barrier-ring self-test (see the header); `result` is a
    device int32 tensor of 3 elements, overwritten."""
    rp = _dev(result, "result", (torch.int32,), 3)
    _check("qlora_selftest_mbarrier_ring",
           lib().qlora_selftest_mbarrier_ring(int(stages), int(consumers), int(iters), int(wait_limit_us), rp,
                                              _stream(stream)))


def qlora_selftest_checks(result, stream=None) -> None:
    """Diagnostic: `result` (device int32, 1 element) becomes QLORA_ERR_CHECK
    (8) when the loaded library was built with the debug checks, else 0."""
    rp = _dev(result, "result", (torch.int32,), 1)
    _check("qlora_selftest_checks", lib().qlora_selftest_checks(rp, _stream(stream)))


def qlora_linear_bwd(w: NF4Weight, X, dY, A, B, r: int, scale: float, dX, accumulate: int, dA, dB, ws,
                     U=None, stream=None) -> None:
    st = w.c_struct()
    M = _tokens(X, "X", w)
    sized = w.numel is not None and _rank_ok(r)
    N, K = w.rows, w.cols
    known = w.numel is not None
    xp = _dev(X, "X", _BF16_BITS)
    gp = _dev(dY, "dY", _BF16_BITS, M * N if known else None)
    ap = _dev(A, "A", _BF16_BITS, r * K if sized else None)
    bp = _dev(B, "B", _BF16_BITS, N * r if sized else None)
    up = _dev_opt(U, "U", _F32, M * r if sized else None)
    dxp = _dev_opt(dX, "dX", _BF16_BITS, M * K if known else None)
    dap = _dev_opt(dA, "dA", _F32, r * K if sized else None)
    dbp = _dev_opt(dB, "dB", _F32, N * r if sized else None)
    wsp, wsb = _ws(ws)
    _check("qlora_linear_bwd",
           lib().qlora_linear_bwd(ctypes.byref(st), xp, gp, M, ap, bp, r, float(scale), up, dxp, int(accumulate), dap,
                                  dbp, wsp, wsb, _stream(stream)))


def qlora_timing_enable(enable: bool) -> None:
    _check("qlora_timing_enable", lib().qlora_timing_enable(1 if enable else 0))


def qlora_timing_read(family: str) -> tuple[float, int]:
    """(summed device milliseconds, launches) of a kernel family since enabling."""
    ms = ctypes.c_double()
    n = ctypes.c_int64()
    _check("qlora_timing_read", lib().qlora_timing_read(family.encode(), ctypes.byref(ms), ctypes.byref(n)))
    return ms.value, n.value
