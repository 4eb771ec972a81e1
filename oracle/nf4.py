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

Variants of the stored format (same steps, other tables):

* FP4 codebook: "FT-02: QLoRA -- Fine-Tuning with Quantization", section
  "Exercise 3: NF4 vs FP4 at equal memory": a floating E2M1 grid (sign bit,
  two exponent bits, one mantissa bit) whose positive levels are printed as
  0, 0.0052, 0.1667, 0.25, 0.3333, 0.5, 0.6667, 1.
* FP8 scale codes: FT-02, section "2c. Double quantization" (the constants
  are quantized in FP8); "QLoRA Deep Dive ...", section "2. Squeezing More
  Memory: Double Quantization (DQ)" (normalize each block of constants by its
  absmax and quantize to 8-bit floats, a standard, not quantile, quantization).
* No double quantization: one fp32 absmax per block, (256 + 32) / 64 = 4.5
  bits per weight ("QLoRA Deep Dive ...", "Memory Savings Analysis"; FT-02
  guided example 3, double quantization on/off).
* 16-bit input weights: FT-02, section "3. BitsAndBytesConfig in practice"
  (each FP16 weight is converted to 4-bit NormalFloat at load time).

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
* FP4 levels: the printed four-digit values are k/12 for k in {0, 1/16, 2, 3,
  4, 6, 8, 12} (0.0052 is 1/192 rounded); the levels are those fractions
  rounded to fp32.  The pages give no bit assignment: code bit 3 is the sign,
  bits 2..0 the magnitude in increasing order (a float's bit pattern orders
  its magnitudes), so code 8 is -0.  The nearest-level rule is NF4's (lowest
  code on a tie), which never picks code 8 and sends ties between two levels
  of one sign to the smaller magnitude.  An odd count is padded with code 0.
* FP8 scale codes: E4M3 (bias 7, three mantissa bits, subnormals, no
  infinities), the normalized value ``fp32(d / c2)`` rounded to the nearest
  E4M3 value, ties to even; code 0 where ``c2 == 0``.  Decoded scale:
  ``a' = fp32(fp32(E4M3(q) * c2) + mu)``.
* 16-bit inputs are widened to fp32 exactly and quantized as fp32.
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

# The FP4 (E2M1) levels in code order: codes 0..7 are the magnitudes k / 12,
# k in {0, 1/16, 2, 3, 4, 6, 8, 12}, ascending; code 8 + c is the negative of
# code c ("FT-02: QLoRA -- Fine-Tuning with Quantization", "Exercise 3: NF4 vs
# FP4 at equal memory").
FP4_TWELFTHS = (0.0, 1.0 / 16.0, 2.0, 3.0, 4.0, 6.0, 8.0, 12.0)
FP4_LEVELS = np.array([F32(k / 12.0) for k in FP4_TWELFTHS] + [-F32(k / 12.0) for k in FP4_TWELFTHS],
                      dtype=np.float32)

CODEBOOKS = {"nf4": NF4_LEVELS, "fp4": FP4_LEVELS}
PAD_CODES = {"nf4": 7, "fp4": 0}  # the +0 level: pad code of an odd count
SCALE_FORMATS = ("dq_int8", "dq_fp8", "fp32")

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


def nearest_level(x: np.ndarray, levels: np.ndarray = NF4_LEVELS) -> np.ndarray:
    """Step Q3: index of the nearest level of each fp32 value.

    ``code = argmin_j |x - L_j|`` with every difference and absolute value in
    fp32, ties going to the lowest index (numpy ``argmin`` returns the first
    minimum), exactly as the teaching quantizer's ``argmin`` over the level
    axis.  ``levels`` is the codebook in code order (NF4 by default).
    Source: "QLoRA: NF4 storage, gradients and local integration", section
    "Exact CPU teaching quantizer and adapter gradient path" (``quantize_nf4``).
    """
    x = np.asarray(x, dtype=F32).ravel()
    levels = np.asarray(levels, dtype=F32)
    out = np.empty(x.size, dtype=np.uint8)
    for s in range(0, x.size, _CHUNK):
        xs = x[s : s + _CHUNK]
        dist = np.abs(xs[:, None] - levels[None, :])  # fp32 array
        out[s : s + _CHUNK] = dist.argmin(axis=1).astype(np.uint8)
    return out


def pack_nibbles(codes: np.ndarray, pad_code: int = ZERO_CODE) -> np.ndarray:
    """Step Q4: two 4-bit codes per byte, element ``2i`` in the low nibble.

    An odd number of codes is padded with the zero level's code (7 for NF4),
    as the teaching quantizer does.  Source: the same section as
    :func:`nearest_level` (the packing of ``quantize_nf4``).
    """
    c = np.asarray(codes, dtype=np.uint8).ravel()
    if c.size % 2:
        c = np.append(c, np.uint8(pad_code))
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


def quantize_nf4(w: np.ndarray, block: int = BLOCK, codebook: str = "nf4"):
    """Steps Q0-Q4: fp32 weights -> (codes, fp32 block absmax, packed bytes).

    Q0 rejects an empty or non-finite input (the teaching quantizer raises
    ``ValueError`` there).  With fp32 input an fp32 absmax can neither
    overflow nor underflow, so its second range guard cannot fire.
    Q1 ``a_b = max |w|`` per block.  Q2 ``x = fp32(w / a_b)``, dividing by 1
    for an all-zero block (the zero-block convention), so that block's codes
    are all the zero level's code and its stored scale is 0.  Q3 nearest
    level of ``codebook`` ("nf4" or "fp4").  Q4 packing.  Source: "QLoRA: NF4
    storage, gradients and local integration", sections "Exact CPU teaching
    quantizer and adapter gradient path" and "NF4: nonuniform reconstruction
    levels" (block of 64); the FP4 levels of "FT-02: QLoRA -- Fine-Tuning
    with Quantization", "Exercise 3: NF4 vs FP4 at equal memory".
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
    codes = nearest_level(x, CODEBOOKS[codebook])
    return codes, absmax, pack_nibbles(codes, PAD_CODES[codebook])


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
    (``P_j``), then the chunk sums left to right in chunk order.  Source:
    "QLoRA: NF4 storage, gradients and local integration", section "Double
    quantization: correct the scale arithmetic" (the stored offset); the
    summation order is this repository's reading of an order the page leaves
    open.
    """
    a = np.asarray(absmax, dtype=F32).ravel()
    nb = a.size
    partials = [sequential_sum_f64(a[j : j + dq_block]) for j in range(0, nb, dq_block)]
    total = sequential_sum_f64(np.array(partials, dtype=np.float64))
    return F32(np.float64(total) / np.float64(nb))


def e4m3_encode(x: np.ndarray) -> np.ndarray:
    """fp32 -> E4M3 codes (uint8), round to nearest, ties to even, saturating.

    E4M3: sign bit, 4 exponent bits (bias 7), 3 mantissa bits; exponent 0
    holds the subnormals m * 2^-9; the largest finite magnitude is 448
    (code 0x7E; 0x7F is NaN; no infinities).  In binade [2^E, 2^(E+1)),
    E >= -6, the spacing is 2^(E-3); below 2^-6 it is 2^-9 (the subnormals
    continue the lowest binade's spacing).  So the magnitude code is
    8 E + 48 + rint(|x| / 2^(E-3)) with E = max(floor(log2 |x|), -6): a
    rounding up to the next power of two carries into the exponent field by
    itself.  Magnitudes past 448 saturate to 0x7E.  The sign bit is the
    input's (-0 gives 0x80).  Source: the FP8 scale codes of "FT-02: QLoRA --
    Fine-Tuning with Quantization", section "2c. Double quantization", read
    as the E4M3 format from its definition.
    """
    x = np.asarray(x, dtype=F32)
    if not np.isfinite(x).all():
        raise ValueError("e4m3_encode takes finite values")
    a = np.abs(x).astype(np.float64)
    _, ex = np.frexp(a)  # a = f 2^ex, f in [0.5, 1)
    E = np.where(a >= 2.0 ** -6, ex - 1, -6).astype(np.int64)
    k = np.rint(np.ldexp(a, -(E - 3)))  # exact scaling; rint is half-to-even
    mag = np.minimum(8 * E + 48 + k.astype(np.int64), 0x7E)
    sign = np.signbit(x).astype(np.int64) << 7
    return (sign | mag).astype(np.uint8)


def e4m3_decode(codes: np.ndarray) -> np.ndarray:
    """E4M3 codes -> fp32 values (exact): (8 + m) 2^(e-10) for e >= 1,
    m 2^-9 for e = 0; NaN for magnitude 0x7F.  Source: as :func:`e4m3_encode`."""
    c = np.asarray(codes, dtype=np.uint8).astype(np.int64)
    e, m = (c >> 3) & 0xF, c & 0x7
    mag = np.where(e == 0, np.ldexp(m.astype(np.float64), -9),
                   np.ldexp((8 + m).astype(np.float64), (e - 10).astype(np.int64)))
    mag = np.where((c & 0x7F) == 0x7F, np.nan, mag)
    return np.where(c >> 7 == 1, -mag, mag).astype(F32)


def double_quantize(absmax: np.ndarray, dq_block: int = DQ_BLOCK, scale_format: str = "dq_int8"):
    """Steps D1-D4: fp32 block scales -> (8-bit codes q, fp32 c2 per chunk, fp32 mu).

    D2 ``d_b = fp32(a_b - mu)``.  D3 ``c2_j = max |d_b|`` over the (possibly
    partial, last) chunk ``j``.  D4, "dq_int8": ``q_b = rint(fp32(fp32(d_b /
    c2_j) * 127))`` with ties to even (int8); "dq_fp8": ``q_b =
    E4M3(fp32(d_b / c2_j))`` (uint8 codes).  ``q_b = 0`` where ``c2_j == 0``.
    Source: "QLoRA: NF4 storage, gradients and local integration", section
    "Double quantization: correct the scale arithmetic"; "QLoRA Deep Dive:
    4-bit NormalFloat & Double Quantization Internals", section "2. Squeezing
    More Memory: Double Quantization (DQ)".
    """
    if scale_format not in ("dq_int8", "dq_fp8"):
        raise ValueError(scale_format)
    a = np.asarray(absmax, dtype=F32).ravel()
    mu = mean_offset(a, dq_block)
    d = (a - mu).astype(F32)
    n_chunks = -(-a.size // dq_block)
    c2 = np.empty(n_chunks, dtype=F32)
    q = np.zeros(a.size, dtype=np.int8 if scale_format == "dq_int8" else np.uint8)
    for j in range(n_chunks):
        dj = d[j * dq_block : (j + 1) * dq_block]
        c = F32(np.max(np.abs(dj)))
        c2[j] = c
        if c != 0:
            ratio = (dj / c).astype(F32)
            if scale_format == "dq_int8":
                scaled = (ratio * F32(127.0)).astype(F32)
                q[j * dq_block : (j + 1) * dq_block] = np.rint(scaled).astype(np.int8)
            else:
                q[j * dq_block : (j + 1) * dq_block] = e4m3_encode(ratio)
    return q, c2, mu


def decode_scales(q: np.ndarray, c2: np.ndarray, mu, dq_block: int = DQ_BLOCK,
                  scale_format: str = "dq_int8") -> np.ndarray:
    """Step R1: ``a'_b = fp32(fp32(t_b * c2_j) + mu)`` with ``t_b = fp32(q_b /
    127)`` ("dq_int8") or the E4M3 value of ``q_b`` ("dq_fp8").  Source: the
    inverse of :func:`double_quantize`, same passages; "QLoRA Deep Dive ...",
    section "The Quantization Process in QLoRA" (decode before use)."""
    c = np.repeat(np.asarray(c2, dtype=F32), dq_block)[: np.asarray(q).size]
    if scale_format == "dq_int8":
        q = np.asarray(q, dtype=np.int8).ravel()
        t = (q.astype(F32) / F32(127.0)).astype(F32)
    elif scale_format == "dq_fp8":
        t = e4m3_decode(np.asarray(q).view(np.uint8).ravel())
    else:
        raise ValueError(scale_format)
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


def dequantize_codes(codes: np.ndarray, scales: np.ndarray, block: int = BLOCK,
                     levels: np.ndarray = NF4_LEVELS) -> np.ndarray:
    """Step R2 in fp32: ``w_hat = fp32(L[code] * a'_b)`` for every code.
    Source: "QLoRA: NF4 storage, gradients and local integration",
    ``dequantize_nf4`` of the teaching program."""
    codes = np.asarray(codes, dtype=np.uint8).ravel()
    per = np.repeat(np.asarray(scales, dtype=F32), block)[: codes.size]
    return (np.asarray(levels, dtype=F32)[codes] * per).astype(F32)


@dataclass
class NF4DQState:
    """The stored state of one quantized tensor (what the library also stores)."""

    shape: tuple
    packed: np.ndarray  # uint8 [n/2]
    qscale: np.ndarray  # int8 (dq_int8) or uint8 E4M3 (dq_fp8) [n/64]; unused for fp32 scales
    c2: np.ndarray  # fp32  [ceil(n/16384)]
    mu: np.float32  # fp32 scalar
    absmax: np.ndarray  # fp32 [n/64] first-level scales (the stored scales for "fp32")
    codebook: str = "nf4"
    scale_format: str = "dq_int8"

    @property
    def n(self) -> int:
        return int(np.prod(self.shape))


def widen_16bit(bits: np.ndarray, dtype: str) -> np.ndarray:
    """16-bit weights (bit patterns, uint16) -> the fp32 values they denote.

    "bf16": the bits are the top half of an fp32; "fp16": IEEE half.  Both
    widenings are exact.  Source: "FT-02: QLoRA -- Fine-Tuning with
    Quantization", section "3. BitsAndBytesConfig in practice" (16-bit
    checkpoints converted at load).
    """
    b = np.asarray(bits, dtype=np.uint16)
    if dtype == "bf16":
        return (b.astype(np.uint32) << 16).view(F32)
    if dtype == "fp16":
        return b.view(np.float16).astype(F32)
    raise ValueError(dtype)


def quantize_weight(w: np.ndarray, codebook: str = "nf4", scale_format: str = "dq_int8") -> NF4DQState:
    """Steps Q0-Q4 then D1-D4 (none for fp32 scales) on one fp32 tensor:
    :func:`quantize_nf4` then :func:`double_quantize`, with their sources."""
    w = np.asarray(w)
    if scale_format not in SCALE_FORMATS:
        raise ValueError(scale_format)
    _, absmax, packed = quantize_nf4(w, codebook=codebook)
    if scale_format == "fp32":
        q, c2, mu = np.zeros(0, dtype=np.int8), np.zeros(0, dtype=F32), F32(0.0)
    else:
        q, c2, mu = double_quantize(absmax, scale_format=scale_format)
    return NF4DQState(tuple(w.shape), packed, q, c2, mu, absmax, codebook, scale_format)


def dequantize_weight(state: NF4DQState, dtype: str = "fp32", double_quant: bool = True) -> np.ndarray:
    """Steps R1-R2: the reconstructed tensor, fp32 values or bf16 bit patterns.

    The state's scale format decides the scale decode; ``double_quant=False``
    uses the fp32 first-level scales of a double-quantized state directly
    (the 4.5-bit storage without double quantization).
    """
    n = state.n
    codes = unpack_nibbles(state.packed, n)
    if state.scale_format == "fp32" or not double_quant:
        scales = state.absmax
    else:
        scales = decode_scales(state.qscale, state.c2, state.mu, scale_format=state.scale_format)
    w_hat = dequantize_codes(codes, scales, levels=CODEBOOKS[state.codebook])[:n].reshape(state.shape)
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


def decision_thresholds(codebook: str = "nf4") -> np.ndarray:
    """The 15 fp32 decision boundaries of :func:`nearest_level` on [-1, 1].

    Let ``order`` list the codes by increasing level (for a tie in value, the
    higher code first) and ``rank(x)`` be the position in ``order`` of
    ``nearest_level(x)``.  ``T_j`` (j = 1..15) is the smallest fp32 value with
    ``rank >= j``, found by bisection over the ordered fp32 bit patterns
    between the levels at positions ``j - 1`` and ``j``.  On that interval
    only those two levels can be nearest (the others are at least one level
    gap away), the rounded distance to the lower one never decreases and the
    one to the upper one never increases as ``x`` grows, so ``rank`` switches
    once: for every fp32 ``x`` in [-1, 1], ``rank(x) = #{ j : x >= T_j }``.
    Two equal levels (FP4's +0 and -0) give ``T_j = T_(j+1)``: the position
    of the one the tie rule never picks is skipped.  For NF4 ``order`` is the
    identity.
    """
    levels = CODEBOOKS[codebook]
    order = sorted(range(16), key=lambda c: (float(levels[c]), -c))
    pos = {c: i for i, c in enumerate(order)}
    out = np.empty(15, dtype=F32)
    for j in range(1, 16):
        lo, hi = _ordered_key(levels[order[j - 1]]), _ordered_key(levels[order[j]])
        if hi == lo:
            # Equal levels: position j - 1 is never chosen, so T_j is the
            # boundary below it; search from the level at position j - 2.
            lo = _ordered_key(levels[order[j - 2]])
        while hi - lo > 1:
            mid = (lo + hi) // 2
            if pos[int(nearest_level(np.array([_from_key(mid)], dtype=F32), levels)[0])] >= j:
                hi = mid
            else:
                lo = mid
        out[j - 1] = _from_key(hi)
    return out
