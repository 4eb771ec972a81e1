"""Pins of the CPU oracle against the pages and against mathematics.

None of these checks re-types the oracle's own formula: each compares it with
a value printed on a page (fixtures under tests/golden/), a closed form, an
independent exact computation (rational arithmetic, brute force) or a library
routine that computes the same quantity another way (torch autograd, scipy's
normal quantile function, torch's bf16 cast).
"""

from fractions import Fraction
import os

import numpy as np
import pytest
import torch

from oracle import accounting, lora, nf4
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


def _figures(golden_dir):
    out = {}
    for line in _read_values(os.path.join(golden_dir, "page_figures.txt")):
        key, val = (s.strip() for s in line.split("=", 1))
        out[key] = float(val)
    return out


# ---------------------------------------------------------------------------
# Codebook
# ---------------------------------------------------------------------------

def test_codebook_matches_printed_table(golden_dir):
    printed = _read_values(os.path.join(golden_dir, "nf4_levels_nf4_storage_page.txt"))
    assert len(printed) == 16
    for j, text in enumerate(printed):
        v = float(text)
        assert float(F32(v)) == v, "each printed level is an exact fp32 value"
        assert float(nf4.NF4_LEVELS[j]) == v


def test_codebook_structure(golden_dir):
    fig = _figures(golden_dir)
    L = nf4.NF4_LEVELS.astype(np.float64)
    assert L.size == 16
    assert (L < 0).sum() == fig["negative_levels"]
    assert (L > 0).sum() == fig["positive_levels"]
    assert L[nf4.ZERO_CODE] == 0.0 and (L == 0).sum() == 1
    assert L[0] == -1.0 and L[15] == 1.0
    assert np.all(np.diff(L) > 0)
    assert not np.allclose(L, -L[::-1]), "the table is asymmetric"
    assert ((L >= -0.2) & (L <= 0.2)).sum() == fig["levels_in_pm02"]


def test_codebook_against_rounded_table(golden_dir):
    rounded = np.array([float(v) for v in _read_values(os.path.join(golden_dir, "nf4_levels_deep_dive_page.txt"))])
    diff = np.abs(rounded - nf4.NF4_LEVELS.astype(np.float64))
    garbled = {3, 8}
    for j in range(16):
        if j in garbled:
            assert diff[j] > 5e-5
        else:
            assert diff[j] <= 5e-5 + 1e-12


def test_codebook_is_normal_quantile_construction():
    # Equal-mass construction: eight positive levels at the standard normal
    # quantiles of evenly spaced probabilities from p0 down to 1/2 (exclusive),
    # seven negative levels likewise, zero added, normalised by the largest.
    # p0 = 1 - (1/32 + 1/30) / 2 is fitted, not printed on the pages.
    from scipy.stats import norm

    p0 = 1.0 - 0.5 * (1.0 / 32 + 1.0 / 30)
    pos = norm.ppf(np.linspace(p0, 0.5, 9)[:-1])
    neg = -norm.ppf(np.linspace(p0, 0.5, 8)[:-1])
    v = np.sort(np.concatenate([pos, [0.0], neg]))
    v /= np.abs(v).max()
    assert np.max(np.abs(v - nf4.NF4_LEVELS)) <= 1e-6


# ---------------------------------------------------------------------------
# Nearest-level decision
# ---------------------------------------------------------------------------

def _exact_nearest(xf32):
    L = [Fraction(float(v)) for v in nf4.NF4_LEVELS]
    x = Fraction(float(xf32))
    d = [abs(x - l) for l in L]
    m = min(d)
    return d.index(m), d


def test_nearest_level_brute_force_exact_rational():
    rng = np.random.default_rng(11)
    x = rng.uniform(-1, 1, 3000).astype(F32)
    x = np.concatenate([x, nf4.NF4_LEVELS, np.array([0.0, -0.0, 1e-40, -1e-40], F32)])
    got = nf4.nearest_level(x)
    for xi, gi in zip(x, got):
        want, d = _exact_nearest(xi)
        if gi != want:
            # only a genuine near-tie may differ: the two exact distances agree
            # to within the fp32 rounding of the differences.
            assert abs(d[gi] - d[want]) <= Fraction(2) ** -24
        assert gi == want or abs(int(gi) - want) == 1


def test_levels_map_to_themselves():
    assert np.array_equal(nf4.nearest_level(nf4.NF4_LEVELS), np.arange(16, dtype=np.uint8))


def test_thresholds_sit_at_midpoints():
    T = nf4.decision_thresholds()
    L = [Fraction(float(v)) for v in nf4.NF4_LEVELS]
    for j in range(1, 16):
        mid = (L[j - 1] + L[j]) / 2
        ulp = Fraction(float(np.spacing(np.abs(T[j - 1]))))
        assert abs(Fraction(float(T[j - 1])) - mid) <= 2 * ulp
        assert nf4.nearest_level(np.array([T[j - 1]]))[0] == j
        below = np.nextafter(T[j - 1], F32(-2.0))
        assert nf4.nearest_level(np.array([below]))[0] == j - 1


def test_step_rule_equals_argmin_near_every_threshold():
    T = nf4.decision_thresholds()
    xs = []
    for t in T:
        u = np.array([t], F32).view(np.uint32)[0].astype(np.int64)
        around = np.arange(-4096, 4097, dtype=np.int64) + u
        xs.append(around.astype(np.uint32).view(F32))
    rng = np.random.default_rng(5)
    xs.append(rng.uniform(-1, 1, 1 << 20).astype(F32))
    x = np.concatenate(xs)
    x = x[np.abs(x) <= 1]
    step = np.searchsorted(T, x, side="right").astype(np.uint8)
    assert np.array_equal(nf4.nearest_level(x), step)


# ---------------------------------------------------------------------------
# Quantize / dequantize (no double quantization)
# ---------------------------------------------------------------------------

def test_teaching_program_shapes(golden_dir):
    fig = _figures(golden_dir)
    w = np.random.default_rng(2).normal(0, 0.2, (8, 8)).astype(F32)
    codes, absmax, packed = nf4.quantize_nf4(w)
    assert packed.size == fig["packed_bytes_8x8"]
    assert absmax.nbytes == fig["scale_bytes_8x8"]
    assert codes.size == 64


def test_zero_tensor_reconstructs_exact_zeros():
    w = np.zeros((3, 7), F32)
    codes, absmax, packed = nf4.quantize_nf4(w)
    assert np.all(codes == nf4.ZERO_CODE) and np.all(packed == 0x77)
    assert np.all(absmax == 0)
    st = nf4.quantize_weight(w)
    assert st.mu == 0 and np.all(st.c2 == 0) and np.all(st.qscale == 0)
    assert np.count_nonzero(nf4.dequantize_weight(st)) == 0
    assert np.count_nonzero(nf4.dequantize_weight(st, double_quant=False)) == 0


def test_codebook_round_trip_block16_and_block64():
    codes, absmax, packed = nf4.quantize_nf4(nf4.NF4_LEVELS, block=16)
    back = nf4.dequantize_codes(nf4.unpack_nibbles(packed, 16), absmax, block=16)
    assert np.array_equal(back, nf4.NF4_LEVELS)
    w = np.tile(nf4.NF4_LEVELS, 4)
    st = nf4.quantize_weight(w)
    assert np.array_equal(nf4.unpack_nibbles(st.packed, 64), np.tile(np.arange(16, dtype=np.uint8), 4))
    assert st.mu == 1.0 and st.c2[0] == 0 and st.qscale[0] == 0
    assert np.array_equal(nf4.dequantize_weight(st), w)


def test_pack_order_low_nibble_first():
    assert np.array_equal(nf4.pack_nibbles(np.array([1, 2, 15, 0], np.uint8)), np.array([0x21, 0x0F], np.uint8))
    assert np.array_equal(nf4.pack_nibbles(np.array([3], np.uint8)), np.array([0x73], np.uint8))


def test_block_scale_and_division():
    # A block whose absmax is a power of two divides exactly: codes are the
    # nearest levels of w / 2^k computed exactly.
    rng = np.random.default_rng(3)
    w = rng.uniform(-1, 1, 64).astype(F32)
    w[17] = F32(-4.0)
    w = w * F32(1.0)
    w[:17] *= F32(4.0)
    codes, absmax, _ = nf4.quantize_nf4(w)
    assert absmax[0] == 4.0
    want = [_exact_nearest(F32(v / 4.0))[0] for v in w]
    assert list(codes) == want


def test_nonfinite_and_empty_rejected():
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.array([1.0, np.nan], F32))
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.array([np.inf], F32))
    with pytest.raises(ValueError):
        nf4.quantize_nf4(np.zeros(0, F32))


def test_subnormal_block():
    w = np.zeros(64, F32)
    w[0] = F32(1e-41)
    w[1] = F32(-5e-42)
    codes, absmax, _ = nf4.quantize_nf4(w)
    assert absmax[0] == F32(1e-41)
    assert codes[0] == 15 and codes[2] == nf4.ZERO_CODE
    assert codes[1] == nf4.nearest_level(np.array([F32(-5e-42) / F32(1e-41)]))[0]


# ---------------------------------------------------------------------------
# Double quantization
# ---------------------------------------------------------------------------

def test_dq_constant_scales_closed_form():
    a = np.full(1000, F32(0.0517), F32)
    q, c2, mu = nf4.double_quantize(a)
    assert mu == F32(0.0517)
    assert np.all(c2 == 0) and np.all(q == 0)
    assert np.all(nf4.decode_scales(q, c2, mu) == F32(0.0517))


def test_dq_two_level_closed_form():
    # Alternating scales 0.25 and 0.0625: mean 0.15625, deviation +-0.09375,
    # so every chunk has c2 = 0.09375 and codes +-127 that decode exactly.
    a = np.tile(np.array([0.25, 0.0625], F32), 512 + 64)
    q, c2, mu = nf4.double_quantize(a)
    assert mu == F32(0.15625)
    assert np.all(c2 == F32(0.09375))
    assert np.all(q[0::2] == 127) and np.all(q[1::2] == -127)
    assert np.array_equal(nf4.decode_scales(q, c2, mu), a)


def test_dq_mean_is_the_mean():
    rng = np.random.default_rng(8)
    for nb in (1, 255, 256, 257, 4099):
        a = (np.abs(rng.normal(0.05, 0.01, nb)) + 1e-4).astype(F32)
        mu = nf4.mean_offset(a)
        exact = Fraction(0)
        for v in a:
            exact += Fraction(float(v))
        exact /= nb
        assert abs(Fraction(float(mu)) - exact) <= Fraction(float(np.spacing(mu)))


def test_dq_partial_last_chunk_and_bound():
    rng = np.random.default_rng(9)
    nb = 3 * 256 + 17
    a = np.abs(rng.normal(0.05, 0.02, nb)).astype(F32)
    q, c2, mu = nf4.double_quantize(a)
    assert c2.size == 4
    d = a.astype(np.float64) - float(mu)
    for j in range(4):
        seg = d[j * 256 : (j + 1) * 256]
        assert abs(float(c2[j]) - np.abs(seg).max()) <= 1e-7 * max(1.0, np.abs(seg).max())
    assert np.all(np.abs(q.astype(int)) <= 127)
    dec = nf4.decode_scales(q, c2, mu).astype(np.float64)
    cj = np.repeat(c2.astype(np.float64), 256)[:nb]
    assert np.all(np.abs(dec - a) <= cj / 254 + 4 * np.spacing(np.float32(a.max())))


def test_dq_sign_convention():
    # Larger-than-mean scales get positive codes.
    a = np.array([1.0, 3.0] * 128, F32)
    q, c2, mu = nf4.double_quantize(a)
    assert mu == 2.0 and c2[0] == 1.0
    assert np.all(q[1::2] == 127) and np.all(q[0::2] == -127)


def test_zero_block_inside_dq_reconstructs_zero():
    case = workloads.tiny_case()
    st = nf4.quantize_weight(case.W.numpy())
    assert st.absmax[0] == 0
    assert np.all(st.packed[:32] == 0x77)
    w_hat = nf4.dequantize_weight(st)
    assert np.all(w_hat.ravel()[:64] == 0)


# ---------------------------------------------------------------------------
# Accounting and the pages' figures
# ---------------------------------------------------------------------------

def test_bits_per_weight(golden_dir):
    fig = _figures(golden_dir)
    assert accounting.bits_per_weight(False) == fig["bits_no_dq"]
    assert accounting.bits_per_weight(True) == fig["bits_dq"]
    saving = accounting.bits_per_weight(False) - accounting.bits_per_weight(True)
    assert saving == fig["dq_saving_bits"]
    assert saving * 7e9 / 8 == fig["dq_saving_bytes_7b"]
    assert round(saving * 70e9 / 8 / 1e9, 3) == fig["dq_saving_gb_70b"]
    assert (32 + 256 * 8) / 256 == fig["dd_bits_per_constant"]
    assert 4096 * 4096 // 64 == fig["dd_blocks_4096x4096"]
    assert 64 * 4 // 8 == fig["payload_bytes_per_block"]


def test_stored_bytes_match_bits():
    for n in (16384, 4096 * 4096, 14336 * 4096):
        bits = accounting.stored_bytes(n) * 8 / n
        assert bits == pytest.approx(accounting.bits_per_weight(True) + 32 / n, abs=1e-12)
        st_bytes = n // 2 + n // 64 + 4 * (n // 16384) + 4
        assert accounting.stored_bytes(n) == st_bytes


def test_opt_quantized_params_and_dq_saving(golden_dir):
    fig = _figures(golden_dir)
    n = sum(p.n * p.k for _, _, p in workloads.opt13b_weight_shapes())
    assert n == fig["opt_quantized_params"]
    assert round(n * 0.373 / 8 / 1e6, 1) == fig["opt_dq_theory_mb"]


def test_adapter_counts(golden_dir):
    fig = _figures(golden_dir)
    shapes7b = [(p.n, p.k) for p in workloads.LAYER7B]
    total = workloads.LAYERS7B * accounting.lora_params(16, shapes7b)
    assert total == fig["adapters_7b_r16"]
    assert round(total * 2 / 1e6, 2) == fig["adapters_7b_r16_bf16_mb"]
    assert round(total * 2 * 4 / 1e6, 2) == fig["adapters_7b_r16_fp32_moments_mb"]
    qv = [(2048, 2048), (2048, 2048)]
    for r, key in ((2, "opt_qv_r2_trainable"), (16, "opt_qv_r16_trainable"), (64, "opt_qv_r64_trainable")):
        assert 24 * accounting.lora_params(r, qv) == fig[key]
        assert 24 * accounting.lora_params(r, qv) == fig["opt_qv_per_r"] * r
    assert accounting.lora_params(16, qv) == fig["opt_qv_per_layer_r16"]
    assert 16 / 8 == fig["lora_scaling_r8_a16"]


# ---------------------------------------------------------------------------
# bf16 rounding
# ---------------------------------------------------------------------------

def test_bf16_rounding_matches_torch():
    rng = np.random.default_rng(4)
    v = rng.normal(0, 1, 100000).astype(F32)
    ties = (rng.integers(0, 1 << 15, 2000).astype(np.uint32) << 16 | 0x8000).view(F32)
    v = np.concatenate([v, ties[np.isfinite(ties)], np.array([0.0, -0.0, 1e-40, 65504.0], F32)])
    want = torch.from_numpy(v).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(nf4.round_to_bf16_bits(v), want)
    back = nf4.bf16_bits_to_f32(want)
    assert np.array_equal(back, torch.from_numpy(v).to(torch.bfloat16).float().numpy())


# ---------------------------------------------------------------------------
# LoRA algebra
# ---------------------------------------------------------------------------

def _small_lora(seed, m=5, n=7, k=9, r=3):
    rng = np.random.default_rng(seed)
    return (rng.normal(size=(m, k)), rng.normal(size=(n, k)), rng.normal(size=(r, k)),
            rng.normal(size=(n, r)), rng.normal(size=(m, n)), 1.7)


def test_merge_identity():
    X, W, A, B, _, s = _small_lora(1)
    Y, _ = lora.lora_forward(X, W, A, B, s)
    merged = X @ (W + s * B @ A).T
    assert np.max(np.abs(Y - merged)) <= 1e-12 * np.max(np.abs(Y))


def test_merge_reproduces_the_two_branch_layer():
    """X merge(W, A, B, s)^T equals the unmerged forward (exact arithmetic)."""
    X, W, A, B, _, s = _small_lora(11)
    Y, _ = lora.lora_forward(X, W, A, B, s)
    assert np.max(np.abs(X @ lora.merge(W, A, B, s).T - Y)) <= 1e-12 * np.max(np.abs(Y))


def test_merge_special_cases():
    X, W, A, B, _, s = _small_lora(12, n=12, k=10, r=3)
    assert np.array_equal(lora.merge(W, A, np.zeros_like(B), s), W)  # B = 0: the base weight
    delta = lora.merge(W, A, B, s) - W
    assert np.linalg.matrix_rank(delta) <= 3  # the update lives in an r-dimensional space


def test_requantizing_a_dequantized_weight_keeps_its_codes():
    """Qhat(Qhat(W)) has Qhat(W)'s codes: every block's largest |value| is
    the decoded scale times a +-1 level, so renormalising returns each level
    to within an ulp, far from any decision threshold."""
    rng = np.random.default_rng(13)
    W = (rng.standard_normal((64, 256)) * 0.02).astype(np.float32)
    st = nf4.quantize_weight(W)
    W_hat = nf4.dequantize_weight(st, "fp32")
    st2 = nf4.quantize_weight(np.asarray(W_hat, dtype=np.float32))
    assert np.array_equal(st2.packed, st.packed)
    # ... while the merged-then-requantized weight moves: Qhat(M) - M != 0.
    A = rng.standard_normal((4, 256)) * 0.02
    B = rng.standard_normal((64, 4)) * 0.02
    M = lora.merge(W_hat, A, B, 2.0).astype(np.float32)
    back = nf4.dequantize_weight(nf4.quantize_weight(M), "fp32")
    err = np.linalg.norm(back - M) / np.linalg.norm(M)
    assert 1e-3 < err < 0.2


def test_gradients_match_autograd():
    X, W, A, B, G, s = _small_lora(2)
    tX, tA, tB = (torch.tensor(a, requires_grad=True) for a in (X, A, B))
    tW = torch.tensor(W)
    y = tX @ tW.T + s * (tX @ tA.T) @ tB.T
    (y * torch.tensor(G)).sum().backward()
    dX, dA, dB, _ = lora.lora_backward(X, G, W, A, B, s)
    np.testing.assert_allclose(dX, tX.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dA, tA.grad.numpy(), rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dB, tB.grad.numpy(), rtol=1e-12, atol=1e-12)


def test_gradients_match_finite_differences():
    X, W, A, B, G, s = _small_lora(3)
    dX, dA, dB, _ = lora.lora_backward(X, G, W, A, B, s)
    rng = np.random.default_rng(30)
    h = 1e-4

    def loss(X_, A_, B_):
        return float(np.sum(G * lora.lora_forward(X_, W, A_, B_, s)[0]))

    for _ in range(3):
        for which, grad in (("X", dX), ("A", dA), ("B", dB)):
            args = {"X": X, "A": A, "B": B}
            d = rng.normal(size=args[which].shape)
            plus = dict(args)
            minus = dict(args)
            plus[which] = args[which] + h * d
            minus[which] = args[which] - h * d
            fd = (loss(plus["X"], plus["A"], plus["B"]) - loss(minus["X"], minus["A"], minus["B"])) / (2 * h)
            assert fd == pytest.approx(float(np.sum(grad * d)), rel=1e-7, abs=1e-9)


def test_zero_b_special_case():
    X, W, A, _, G, s = _small_lora(4)
    B = np.zeros((W.shape[0], A.shape[0]))
    Y, _ = lora.lora_forward(X, W, A, B, s)
    assert np.array_equal(Y, X @ W.T)
    dX, dA, dB, _ = lora.lora_backward(X, G, W, A, B, s)
    assert np.count_nonzero(dA) == 0
    assert np.abs(dB).sum() > 0
    assert np.abs(dX).sum() > 0


def test_row_and_adapter_helpers_agree():
    X, W, A, B, G, s = _small_lora(5)
    Y, _ = lora.lora_forward(X, W, A, B, s)
    dX, dA, dB, _ = lora.lora_backward(X, G, W, A, B, s)
    rows = [0, 3]
    np.testing.assert_allclose(lora.lora_forward_rows(rows, X, W, A, B, s), Y[rows], rtol=1e-13)
    np.testing.assert_allclose(lora.lora_backward_rows(rows, G, W, A, B, s), dX[rows], rtol=1e-13)
    ga, gb = lora.lora_adapter_grads(X, G, A, B, s)
    np.testing.assert_allclose(ga, dA, rtol=1e-13)
    np.testing.assert_allclose(gb, dB, rtol=1e-13)


# ---------------------------------------------------------------------------
# Reconstruction error (diagnostic range from the pages)
# ---------------------------------------------------------------------------

def test_reconstruction_error_range():
    # "FT-02 ...", exercise 1: relative Frobenius errors of order 1e-2 to 1e-1.
    w = workloads.normal_f32((256, 1024), 0.02, 12).numpy()
    st = nf4.quantize_weight(w)
    e_dq = np.linalg.norm(nf4.dequantize_weight(st) - w) / np.linalg.norm(w)
    e_nodq = np.linalg.norm(nf4.dequantize_weight(st, double_quant=False) - w) / np.linalg.norm(w)
    assert 1e-2 < e_nodq < 1e-1 and 1e-2 < e_dq < 1e-1
    assert abs(e_dq - e_nodq) / e_nodq < 0.01


def test_exact_ties_go_to_the_lower_level():
    # Where the midpoint of two adjacent levels is an fp32 value, both rounded
    # distances are equal there; numpy's argmin (the teaching quantizer's rule)
    # returns the lower index.
    L = [Fraction(float(v)) for v in nf4.NF4_LEVELS]
    found = 0
    for j in range(1, 16):
        mid = (L[j - 1] + L[j]) / 2
        m32 = F32(float(mid))
        if Fraction(float(m32)) != mid:
            continue
        found += 1
        assert nf4.nearest_level(np.array([m32]))[0] == j - 1
        assert nf4.nearest_level(np.array([np.nextafter(m32, F32(2))]))[0] == j
    assert found >= 1


def _dq_tie_scales():
    """One chunk of 256 block scales 256 +- d for d = 127 and every
    half-integer k + 1/2 (k = 0 .. 126): the mean is exactly 256, every
    deviation d_b = a_b - mu is exact, c2 = 127, and d / c2 * 127 gives back
    d exactly in fp32 for all of them (checked here), so each half-integer
    deviation lands exactly on a rounding tie of step D4."""
    d = np.array([127.0] + [k + 0.5 for k in range(127)], F32)
    a = np.empty(256, F32)
    a[0::2] = F32(256.0) + d
    a[1::2] = F32(256.0) - d
    for v in d[1:]:
        for sv in (v, -v):
            assert F32(F32(F32(sv) / F32(127.0)) * F32(127.0)) == F32(sv)  # an exact tie reaches D4
    return a, d


def test_dq_rounding_ties_go_to_even():
    """Step D4 rounds to nearest with ties to even: a deviation of exactly
    k + 1/2 code steps gives the even one of k and k + 1 (0.5 -> 0, 1.5 -> 2,
    2.5 -> 2, and the same magnitudes with the sign for negative deviations).
    Rounding half away from zero, or truncation, fails here."""
    a, d = _dq_tie_scales()
    q, c2, mu = nf4.double_quantize(a)
    assert mu == F32(256.0) and c2[0] == F32(127.0)
    assert q[0] == 127 and q[1] == -127
    for i, k in enumerate(range(127), start=1):
        want = k if k % 2 == 0 else k + 1  # the even neighbour of k + 1/2
        assert q[2 * i] == want, (k, q[2 * i])
        assert q[2 * i + 1] == -want, (k, q[2 * i + 1])
    assert [int(v) for v in q[2:8]] == [0, 0, 2, -2, 2, -2]  # 0.5, 1.5, 2.5 and their negatives
