"""Pins of the oracle's format variants: the FP4 codebook, E4M3 scale codes,
fp32 scales (no double quantization) and 16-bit input weights.

As for the NF4 pins, no check re-types the oracle's formula: each compares it
with values printed on a page (tests/golden/), exact rational arithmetic,
brute force, or a library routine computing the same thing another way
(torch's float8_e4m3fn, bf16 and fp16 casts).
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

from oracle import accounting, nf4
from bit_nf4_quantized_blk_b200 import workloads

F32 = np.float32


def _read_values(path):
    vals = []
    with open(path) as f:
        for line in f:
            line = line.split("#", 1)[0].strip()
            if line:
                vals.append(line)
    return vals


# ---------------------------------------------------------------------------
# FP4 codebook
# ---------------------------------------------------------------------------

def test_fp4_levels_match_the_printed_values(golden_dir):
    printed = [float(v) for v in _read_values(os.path.join(golden_dir, "fp4_levels_ft02_page.txt"))]
    pos = [float(v) for v in nf4.FP4_LEVELS[:8]]
    assert len(printed) == 8
    for p, v in zip(printed, pos):
        assert abs(p - v) <= 0.5e-4 + 1e-12, (p, v)  # the page rounds to four decimals


def test_fp4_sign_magnitude_layout():
    L = nf4.FP4_LEVELS
    # bit 3 is the sign: codes 8..15 negate codes 0..7 (code 8 is -0)
    assert np.array_equal(L[8:], -L[:8])
    assert np.signbit(L[8]) and L[8] == 0 and not np.signbit(L[0])
    # magnitudes increase with the code, from 0 to 1
    assert np.all(np.diff(L[:8]) > 0) and L[0] == 0 and L[7] == 1
    # same 4 bits per weight as NF4: the codebook changes no storage size
    assert L.size == nf4.NF4_LEVELS.size == 16


def test_fp4_levels_are_twelfths_in_fp32():
    # 12 * level is 0, 1/16, 2, 3, 4, 6, 8, 12 up to fp32 rounding (exact rationals)
    want = [Fraction(0), Fraction(1, 16), 2, 3, 4, 6, 8, 12]
    for v, k in zip(nf4.FP4_LEVELS[:8], want):
        assert abs(Fraction(float(v)) * 12 - k) <= Fraction(12) * Fraction(float(np.spacing(F32(abs(v)) or F32(1e-38)))), (v, k)


def _exact_nearest_codes(x, levels):
    xf = Fraction(float(x))
    d = [abs(xf - Fraction(float(l))) for l in levels]
    m = min(d)
    return [i for i, v in enumerate(d) if v == m], d


def test_fp4_nearest_level_brute_force_exact_rational():
    rng = np.random.default_rng(21)
    x = np.concatenate([rng.uniform(-1, 1, 3000).astype(F32), rng.uniform(-0.01, 0.01, 500).astype(F32),
                        nf4.FP4_LEVELS, np.array([0.0, -0.0, 1e-40, -1e-40], F32)])
    got = nf4.nearest_level(x, nf4.FP4_LEVELS)
    L = nf4.FP4_LEVELS
    for xi, gi in zip(x, got):
        ties, d = _exact_nearest_codes(xi, L)
        if gi in ties:
            assert gi == min(ties)  # lowest code among exact ties (e.g. +0 over -0)
        else:
            # a genuine near-tie only: the exact distances agree to the fp32 rounding
            assert min(abs(d[gi] - d[t]) for t in ties) <= Fraction(2) ** -24


def test_fp4_never_emits_negative_zero():
    codes = nf4.nearest_level(np.array([0.0, -0.0, -1e-30, -0.001, 1e-30], F32), nf4.FP4_LEVELS)
    assert np.array_equal(codes, np.zeros(5, np.uint8))
    # No two same-sign FP4 levels have an fp32 midpoint (each needs more
    # than 24 significant bits), so +0 / -0 is the only exact tie.
    L = nf4.FP4_LEVELS
    for sign in (0, 8):
        for c in range(1, 7):
            mid = (Fraction(float(L[sign + c])) + Fraction(float(L[sign + c + 1]))) / 2
            assert Fraction(float(F32(float(mid)))) != mid


@pytest.mark.parametrize("codebook", ["nf4", "fp4"])
def test_threshold_rule_equals_argmin_near_every_threshold(codebook):
    levels = nf4.CODEBOOKS[codebook]
    T = nf4.decision_thresholds(codebook)
    order = sorted(range(16), key=lambda c: (float(levels[c]), -c))
    assert np.all(np.diff(T) >= 0)
    xs = []
    for t in T:
        u = np.array([t], F32).view(np.uint32)[0].astype(np.int64)
        xs.append((np.arange(-2048, 2049, dtype=np.int64) + u).astype(np.uint32).view(F32))
    xs.append(np.random.default_rng(6).uniform(-1, 1, 1 << 18).astype(F32))
    xs.append(np.array([0.0, -0.0, 1.0, -1.0], F32))
    x = np.concatenate(xs)
    x = x[np.abs(x) <= 1]
    rank = np.searchsorted(T, x, side="right")
    assert np.array_equal(nf4.nearest_level(x, levels), np.array(order, np.uint8)[rank])


def test_nf4_beats_fp4_on_gaussian_weights():
    """The page expects NF4's quantile grid to reconstruct normally distributed
    weights better than FP4 at equal memory (a prediction, checked here on a
    large synthetic sample)."""
    W = workloads.normal_f32((512, 4096), 0.02, 77).numpy()
    err = {}
    for cb in ("nf4", "fp4"):
        st = nf4.quantize_weight(W, codebook=cb, scale_format="fp32")
        err[cb] = float(np.mean((nf4.dequantize_weight(st) - W).astype(np.float64) ** 2))
    assert err["nf4"] < err["fp4"]


def test_fp4_round_trip_and_zero_block():
    st = nf4.quantize_weight(np.outer(np.ones(2, F32), np.resize(nf4.FP4_LEVELS, 64)).astype(F32), codebook="fp4",
                             scale_format="fp32")
    codes = nf4.unpack_nibbles(st.packed, 128)
    want = np.resize(np.arange(16, dtype=np.uint8), 64)
    want[want == 8] = 0  # -0 comes back as +0
    assert np.array_equal(codes, np.concatenate([want, want]))
    z = nf4.quantize_weight(np.zeros((1, 64), F32), codebook="fp4", scale_format="fp32")
    assert np.all(z.packed == 0) and np.all(nf4.dequantize_weight(z) == 0)


# ---------------------------------------------------------------------------
# E4M3 scale codes
# ---------------------------------------------------------------------------

def _torch_e4m3(x):
    return torch.from_numpy(np.asarray(x, F32)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def test_e4m3_anchor_codes():
    x = np.array([448.0, 1.0, 2.0 ** -6, 2.0 ** -9, 0.0, -0.0, -1.0, 0.875, 240.0], F32)
    assert nf4.e4m3_encode(x).tolist() == [0x7E, 0x38, 0x08, 0x01, 0x00, 0x80, 0xB8, 0x36, 0x77]
    assert np.isnan(nf4.e4m3_decode(np.array([0x7F, 0xFF], np.uint8))).all()


def test_e4m3_decode_matches_torch_for_every_code():
    codes = np.arange(256, dtype=np.uint8)
    ours = nf4.e4m3_decode(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    finite = ~np.isnan(ref)
    assert np.array_equal(np.isnan(ours), ~finite)
    assert np.array_equal(ours[finite].view(np.uint32), ref[finite].view(np.uint32))


def test_e4m3_encode_matches_torch_rne():
    vals = nf4.e4m3_decode(np.arange(0x7F, dtype=np.uint8)).astype(np.float64)  # 0 .. 448
    mids = (vals[:-1] + vals[1:]) / 2  # exact ties: round half to even
    rng = np.random.default_rng(9)
    xs = np.concatenate([vals, mids, np.nextafter(mids.astype(F32), F32(0)), np.nextafter(mids.astype(F32), F32(1e9)),
                         rng.uniform(-1, 1, 20000), rng.uniform(-2.0 ** -6, 2.0 ** -6, 5000),
                         rng.uniform(-448, 448, 5000)]).astype(F32)
    xs = np.concatenate([xs, -xs])
    assert np.array_equal(nf4.e4m3_encode(xs), _torch_e4m3(xs))
    # every finite code round-trips
    codes = np.array([c for c in range(256) if c & 0x7F != 0x7F], np.uint8)
    assert np.array_equal(nf4.e4m3_encode(nf4.e4m3_decode(codes)), codes)


def test_e4m3_saturates_and_rejects_nonfinite():
    assert nf4.e4m3_encode(np.array([1e6, -500.0], F32)).tolist() == [0x7E, 0xFE]
    with pytest.raises(ValueError):
        nf4.e4m3_encode(np.array([np.inf], F32))


def test_fp8_scales_error_bound_and_comparison_with_int8():
    """Decoded E4M3 scales lie within half an E4M3 spacing of the true scale:
    |a' - a| <= c2 max(2^-4 |d / c2|, 2^-10) plus the fp32 roundings; int8
    codes are within c2 / 254.  On Gaussian weights the int8 codes have the
    smaller worst-case error, the E4M3 codes the smaller error on the small
    deviations."""
    W = workloads.normal_f32((256, 4096), 0.02, 3).numpy()
    a = nf4.quantize_weight(W, scale_format="fp32").absmax.astype(np.float64)
    errs = {}
    for fmt in ("dq_int8", "dq_fp8"):
        q, c2, mu = nf4.double_quantize(a.astype(F32), scale_format=fmt)
        dec = nf4.decode_scales(q, c2, mu, scale_format=fmt).astype(np.float64)
        cc = np.repeat(c2.astype(np.float64), 256)[: a.size]
        d = a - np.float64(mu)
        if fmt == "dq_fp8":
            bound = cc * np.maximum(2.0 ** -4 * np.abs(d / cc), 2.0 ** -10) + 4 * 2.0 ** -24 * (np.abs(a) + cc)
        else:
            bound = cc / 254 + 4 * 2.0 ** -24 * (np.abs(a) + cc)
        assert np.all(np.abs(dec - a) <= bound), fmt
        errs[fmt] = np.abs(dec - a)
    assert errs["dq_int8"].max() < errs["dq_fp8"].max()
    small = np.abs(a - a.mean()) < 0.05 * np.abs(a - a.mean()).max()
    assert errs["dq_fp8"][small].mean() < errs["dq_int8"][small].mean()


def test_fp8_dq_zero_chunk_and_storage():
    a = np.full(300, 0.5, F32)
    q, c2, mu = nf4.double_quantize(a, scale_format="dq_fp8")
    assert q.dtype == np.uint8 and np.all(q == 0) and np.all(c2 == 0) and mu == F32(0.5)
    assert np.array_equal(nf4.decode_scales(q, c2, mu, scale_format="dq_fp8"), a)
    # same bytes as the int8 codes: one per block
    assert accounting.bits_per_weight(True) == pytest.approx(4.126953125)


# ---------------------------------------------------------------------------
# fp32 scales (no double quantization) and 16-bit inputs
# ---------------------------------------------------------------------------

def test_fp32_scales_reconstruct_with_the_block_absmax():
    W = workloads.normal_f32((8, 128), 0.02, 4).numpy()
    st = nf4.quantize_weight(W, scale_format="fp32")
    blocks = W.reshape(-1, 64)
    assert np.array_equal(st.absmax, np.abs(blocks).max(axis=1))
    codes = nf4.unpack_nibbles(st.packed, W.size).reshape(-1, 64)
    want = (nf4.NF4_LEVELS[codes] * st.absmax[:, None]).astype(F32)
    assert np.array_equal(nf4.dequantize_weight(st).reshape(-1, 64), want)
    assert accounting.bits_per_weight(False) == 4.5


def test_widen_16bit_matches_torch_casts():
    rng = np.random.default_rng(12)
    bits = np.concatenate([rng.integers(0, 1 << 16, 20000), [0x0000, 0x8000, 0x0001, 0x3F80, 0x3C00, 0x7BFF]])
    bits = bits.astype(np.uint16)
    bf = torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).float().numpy()
    hf = torch.from_numpy(bits.view(np.int16)).view(torch.float16).float().numpy()
    for name, ref in (("bf16", bf), ("fp16", hf)):
        ours = nf4.widen_16bit(bits, name)
        fin = np.isfinite(ref)
        assert np.array_equal(ours[fin].view(np.uint32), ref[fin].view(np.uint32)), name
    assert nf4.widen_16bit(np.array([0x3C00], np.uint16), "fp16")[0] == 1.0
    assert nf4.widen_16bit(np.array([0x0001], np.uint16), "fp16")[0] == F32(2.0 ** -24)


@pytest.mark.parametrize("codebook", ["nf4", "fp4"])
@pytest.mark.parametrize("scale_format", ["dq_int8", "dq_fp8", "fp32"])
def test_format_variants_reconstruct_within_the_grid(codebook, scale_format):
    """Every reconstructed weight lies within half the widest level gap of its
    block scale from the input, and within the scale error."""
    W = workloads.normal_f32((16, 256), 0.02, 8).numpy()
    st = nf4.quantize_weight(W, codebook=codebook, scale_format=scale_format)
    w_hat = nf4.dequantize_weight(st).astype(np.float64)
    L = np.sort(nf4.CODEBOOKS[codebook].astype(np.float64))
    half_gap = np.max(np.diff(L)) / 2
    a = np.repeat(st.absmax.astype(np.float64), 64).reshape(W.shape)
    if scale_format == "fp32":
        scale_err = 0
    else:
        dec = np.repeat(nf4.decode_scales(st.qscale, st.c2, st.mu, scale_format=scale_format), 64).reshape(W.shape)
        scale_err = np.abs(dec.astype(np.float64) - a)
    assert np.all(np.abs(w_hat - W) <= half_gap * a + scale_err + 1e-9)
