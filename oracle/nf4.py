"""NF4 blockwise quantization, double quantization and dequantization (oracle).

Test infrastructure: only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may use this module.

Each function follows one step of the method as the pages give it:

* Codebook: the 16 NF4 levels printed in "QLoRA: NF4 storage, gradients and
  local integration", section "Exact CPU teaching quantizer and adapter
  gradient path" (the ``NF4`` array).  Seven negative levels, an exact zero,
  eight positive levels, endpoints -1 and +1 (same page, section "NF4:
  nonuniform reconstruction levels").
* Quantize (steps Q0-Q4): per block of 64 consecutive weights of the
  row-major flattening, take the absolute maximum, divide every weight by it
  (an all-zero block divides by 1), pick the nearest level (lowest index on a
  tie, as numpy's ``argmin``), pack two 4-bit codes per byte with the even
  element in the low nibble; an odd count is padded with code 7.  Same page
  and section (``quantize_nf4``); block size from section "NF4: nonuniform
  reconstruction levels".
* Double quantization (steps D1-D4): the fp32 block scales are quantized to
  8 bits in chunks of 256 with one fp32 second-level absmax per chunk, after
  subtracting a stored per-tensor offset.  Same page, section "Double
  quantization: correct the scale arithmetic"; "QLoRA Deep Dive: 4-bit
  NormalFloat & Double Quantization Internals", section "2. Squeezing More
  Memory: Double Quantization (DQ)" (absmax per 256 constants becomes the
  second-level constant; a standard, not quantile, 8-bit quantization).
* Dequantize (steps R1-R2): decode the block scale, multiply the level by it,
  cast to the compute dtype.  "QLoRA Deep Dive ...", section "The
  Quantization Process in QLoRA"; "QLoRA: NF4 storage ...", ``dequantize_nf4``.

Readings of what the pages leave open (each is also listed in the design
notes of the repository):

* Arithmetic precision of the normalisation and of the nearest-level search:
  fp32 with IEEE round-to-nearest-even (the teaching code uses float64; the
  library contract fixes fp32).  The distances ``|x - L_j|`` are rounded to
  fp32 before the comparison.
* The 8-bit scale format: symmetric linear int8 in [-127, 127] around a
  per-tensor mean offset, ``q = rint(127 * d / c2)`` with ties to even;
  ``q = 0`` where ``c2 == 0``.
* The per-tensor mean ``mu`` is accumulated in fp64, strictly sequentially:
  first inside each chunk of 256 block scales, then over the chunk sums in
  chunk order; ``mu = fp32(S / nb)``.
* Decoded scale: ``a' = fp32(fp32(fp32(q / 127) * c2) + mu)``, three rounded
  operations in that order, no fused multiply-add.
* Dequantized weight: ``w_hat = fp32(L[code] * a')``; the bf16 output is that
  value rounded to nearest even.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np

F32 = np.float32

# The 16 NF4 levels, as printed (decimal) on "QLoRA: NF4 storage, gradients and
# local integration", section "Exact CPU teaching quantizer and adapter gradient
# path".  Every entry is exactly representable in fp32.
NF4_LEVELS = np.array(
    [
        -1.0,
        -0.6961928009986877,
        -0.5250730514526367,
        -0.39491748809814453,
        -0.28444138169288635,
        -0.18477343022823334,
        -0.09105003625154495,
        0.0,
        0.07958029955625534,
        0.16093020141124725,
        0.24611230194568634,
        0.33791524171829224,
        0.44070982933044434,
        0.5626170039176941,
        0.7229568362236023,
        1.0,
    ],
    dtype=np.float32,
)

BLOCK = 64  # weights per first-level block
DQ_BLOCK = 256  # first-level scales per double-quant chunk
ZERO_CODE = 7  # index of the exact 0.0 level; also the odd-count pad code

_CHUNK = 1 << 20  # elements per slice of the nearest-level search (memory only)


def assert_ieee_subnormals() -> None:
    """Refuse to run if the host FPU flushes subnormals (FTZ/DAZ).

    Every step here relies on IEEE fp32 with gradual underflow; a library that
    switched the process to flush-to-zero would silently change codes.
    """
    tiny = np.array([1.0e-45], dtype=F32)
    if not (tiny * F32(1.0))[0] > 0 or not (tiny[0] / F32(2.0)) >= 0:
        raise RuntimeError("host FPU flushes fp32 subnormals; oracle results would be wrong")
    if np.float32(np.float32(2.0 ** -140) * np.float32(0.5)) == 0:
        raise RuntimeError("host FPU flushes fp32 subnormals; oracle results would be wrong")


def nearest_level(x: np.ndarray) -> np.ndarray:
    """Step Q3: index of the nearest NF4 level of each fp32 value.

    ``code = argmin_j |x - L_j|`` with every difference and absolute value in
    fp32, ties going to the lowest index (numpy ``argmin`` returns the first
    minimum), exactly as the teaching quantizer's ``argmin`` over the level
    axis.
    """
    x = np.asarray(x, dtype=F32).ravel()
    out = np.empty(x.size, dtype=np.uint8)
    for s in range(0, x.size, _CHUNK):
        xs = x[s : s + _CHUNK]
        dist = np.abs(xs[:, None] - NF4_LEVELS[None, :])  # fp32 array
        out[s : s + _CHUNK] = dist.argmin(axis=1).astype(np.uint8)
    return out


def pack_nibbles(codes: np.ndarray) -> np.ndarray:
    """Step Q4: two 4-bit codes per byte, element ``2i`` in the low nibble.

    An odd number of codes is padded with code 7 (the zero level), as the
    teaching quantizer does.
    """
    c = np.asarray(codes, dtype=np.uint8).ravel()
    if c.size % 2:
        c = np.append(c, np.uint8(ZERO_CODE))
    return (c[0::2] | (c[1::2] << 4)).astype(np.uint8)


def unpack_nibbles(packed: np.ndarray, count: int) -> np.ndarray:
    """Inverse of :func:`pack_nibbles`: the first ``count`` codes."""
    p = np.asarray(packed, dtype=np.uint8).ravel()
    codes = np.empty(2 * p.size, dtype=np.uint8)
    codes[0::2] = p & 0x0F
    codes[1::2] = p >> 4
    return codes[:count]


def blocks_of(w: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Row-major flattening, zero-padded to a multiple of ``block``, as rows."""
    flat = np.asarray(w, dtype=F32).ravel()
    pad = (-flat.size) % block
    if pad:
        flat = np.concatenate([flat, np.zeros(pad, dtype=F32)])
    return flat.reshape(-1, block)


def quantize_nf4(w: np.ndarray, block: int = BLOCK):
    """Steps Q0-Q4: fp32 weights -> (codes, fp32 block absmax, packed bytes).

    Q0 rejects an empty or non-finite input (the teaching quantizer raises
    ``ValueError`` there).  With fp32 input an fp32 absmax can neither
    overflow nor underflow, so its second range guard cannot fire.
    Q1 ``a_b = max |w|`` per block.  Q2 ``x = fp32(w / a_b)``, dividing by 1
    for an all-zero block (the zero-block convention), so that block's codes
    are all 7 and its stored scale is 0.  Q3 nearest level.  Q4 packing.
    """
    assert_ieee_subnormals()
    w = np.asarray(w)
    if w.dtype != F32:
        raise TypeError("the quantizer takes fp32 weights")
    if w.size == 0 or block < 1:
        raise ValueError("quantizer input must be non-empty")
    if not np.isfinite(w).all():
        raise ValueError("quantizer input must be finite")
    blocks = blocks_of(w, block)
    absmax = np.max(np.abs(blocks), axis=1).astype(F32)
    divisor = np.where(absmax == 0, F32(1.0), absmax).astype(F32)
    x = (blocks / divisor[:, None]).astype(F32)
    codes = nearest_level(x)
    return codes, absmax, pack_nibbles(codes)


def sequential_sum_f64(values: np.ndarray) -> float:
    """fp64 sum taken strictly left to right (each partial rounded to fp64).

    ``np.add.accumulate`` computes ``out[i] = out[i-1] + v[i]`` in order, so
    its last element is the left-to-right sum.
    """
    v = np.asarray(values, dtype=np.float64).ravel()
    if v.size == 0:
        return 0.0
    return float(np.add.accumulate(v)[-1])


def mean_offset(absmax: np.ndarray, dq_block: int = DQ_BLOCK) -> np.float32:
    """Step D1: ``mu = fp32(S / nb)``, the per-tensor mean of the block scales.

    ``S`` is summed in fp64: first the 256 scales of each chunk left to right
    (``P_j``), then the chunk sums left to right in chunk order.
    """
    a = np.asarray(absmax, dtype=F32).ravel()
    nb = a.size
    partials = [sequential_sum_f64(a[j : j + dq_block]) for j in range(0, nb, dq_block)]
    total = sequential_sum_f64(np.array(partials, dtype=np.float64))
    return F32(np.float64(total) / np.float64(nb))


def double_quantize(absmax: np.ndarray, dq_block: int = DQ_BLOCK):
    """Steps D1-D4: fp32 block scales -> (int8 codes q, fp32 c2 per chunk, fp32 mu).

    D2 ``d_b = fp32(a_b - mu)``.  D3 ``c2_j = max |d_b|`` over the (possibly
    partial, last) chunk ``j``.  D4 ``q_b = rint(fp32(fp32(d_b / c2_j) * 127))``
    with ties to even, or 0 where ``c2_j == 0``.
    """
    a = np.asarray(absmax, dtype=F32).ravel()
    mu = mean_offset(a, dq_block)
    d = (a - mu).astype(F32)
    n_chunks = -(-a.size // dq_block)
    c2 = np.empty(n_chunks, dtype=F32)
    q = np.zeros(a.size, dtype=np.int8)
    for j in range(n_chunks):
        dj = d[j * dq_block : (j + 1) * dq_block]
        c = F32(np.max(np.abs(dj)))
        c2[j] = c
        if c != 0:
            ratio = (dj / c).astype(F32)
            scaled = (ratio * F32(127.0)).astype(F32)
            q[j * dq_block : (j + 1) * dq_block] = np.rint(scaled).astype(np.int8)
    return q, c2, mu


def decode_scales(q: np.ndarray, c2: np.ndarray, mu, dq_block: int = DQ_BLOCK) -> np.ndarray:
    """Step R1: ``a'_b = fp32(fp32(fp32(q_b / 127) * c2_j) + mu)``."""
    q = np.asarray(q, dtype=np.int8).ravel()
    c = np.repeat(np.asarray(c2, dtype=F32), dq_block)[: q.size]
    t = (q.astype(F32) / F32(127.0)).astype(F32)
    t = (t * c).astype(F32)
    return (t + F32(mu)).astype(F32)


def round_to_bf16_bits(values: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns, round to nearest, ties to even (finite inputs)."""
    u = np.asarray(values, dtype=F32).view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    return ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> the fp32 values they denote (exact)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(F32)


def dequantize_codes(codes: np.ndarray, scales: np.ndarray, block: int = BLOCK) -> np.ndarray:
    """Step R2 in fp32: ``w_hat = fp32(L[code] * a'_b)`` for every code."""
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    per = np.repeat(np.asarray(scales, dtype=F32), block)[: codes.size]
    return (NF4_LEVELS[codes] * per).astype(F32)


@dataclass
class NF4DQState:
    """The stored state of one quantized tensor (what the library also stores)."""

    shape: tuple
    packed: np.ndarray  # uint8 [n/2]
    qscale: np.ndarray  # int8  [n/64]
    c2: np.ndarray  # fp32  [ceil(n/16384)]
    mu: np.float32  # fp32 scalar
    absmax: np.ndarray  # fp32 [n/64] first-level scales (kept for diagnostics)

    @property
    def n(self) -> int:
        return int(np.prod(self.shape))


def quantize_weight(w: np.ndarray) -> NF4DQState:
    """Steps Q0-Q4 then D1-D4 on one tensor."""
    w = np.asarray(w)
    _, absmax, packed = quantize_nf4(w)
    q, c2, mu = double_quantize(absmax)
    return NF4DQState(tuple(w.shape), packed, q, c2, mu, absmax)


def dequantize_weight(state: NF4DQState, dtype: str = "fp32", double_quant: bool = True) -> np.ndarray:
    """Steps R1-R2: the reconstructed tensor, fp32 values or bf16 bit patterns.

    ``double_quant=False`` uses the fp32 first-level scales directly (the
    4.5-bit storage without double quantization).
    """
    n = state.n
    codes = unpack_nibbles(state.packed, n)
    scales = decode_scales(state.qscale, state.c2, state.mu) if double_quant else state.absmax
    w_hat = dequantize_codes(codes, scales)[:n].reshape(state.shape)
    if dtype == "fp32":
        return w_hat
    if dtype == "bf16":
        return round_to_bf16_bits(w_hat)
    raise ValueError(dtype)


def _ordered_key(f: np.float32) -> int:
    u = int(np.asarray(f, dtype=F32).view(np.uint32))
    return (u & 0x7FFFFFFF) if u >> 31 == 0 else -(u & 0x7FFFFFFF)


def _from_key(k: int) -> np.float32:
    u = k if k >= 0 else (0x80000000 | -k)
    return np.array([u], dtype=np.uint32).view(F32)[0]


def decision_thresholds() -> np.ndarray:
    """The 15 fp32 decision boundaries of :func:`nearest_level` on [-1, 1].

    ``T_j`` (j = 1..15) is the smallest fp32 value whose nearest level has
    index ``j``, found by bisection over the ordered fp32 bit patterns between
    ``L[j-1]`` and ``L[j]``.  On that interval only those two levels can be
    nearest (the other levels are at least one level gap away), the rounded
    distance to ``L[j-1]`` never decreases and the one to ``L[j]`` never
    increases as ``x`` grows, so the choice switches once: for every fp32
    ``x`` in [-1, 1], ``nearest_level(x) = #{ j : x >= T_j }``.
    """
    out = np.empty(15, dtype=F32)
    for j in range(1, 16):
        lo, hi = _ordered_key(NF4_LEVELS[j - 1]), _ordered_key(NF4_LEVELS[j])
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if nearest_level(np.array([_from_key(mid)], dtype=F32))[0] >= j:
                hi = mid
            else:
                lo = mid
        out[j - 1] = _from_key(hi)
    return out
