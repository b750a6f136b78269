"""Pins of the oracle's LayerNorm + adaLN modulate before the quantize
(reading R19: population variance, eps inside the square root, no affine
LayerNorm parameters, m = h * (1 + scale) + shift), against a float64 numpy
LayerNorm, exact rational statistics and closed-form rows."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_video_dit_b200 import synthetic as syn


def _ln64(x, scale, shift, eps):
    mu = x.mean(axis=1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=1, keepdims=True)
    h = (x - mu) / np.sqrt(var + eps)
    return h * (1.0 + scale) + shift


@pytest.mark.parametrize("rows,cols", [(64, 3072), (5, 64), (3, 1040)])
def test_matches_float64_layernorm_modulate(rows, cols):
    bits = syn.activations_bf16(rows, cols, seed=rows + cols)
    sc = syn.normal_bf16((cols,), seed=1, std=0.1)
    sh = syn.normal_bf16((cols,), seed=2, std=0.1)
    m = oracle.ln_modulate(bits, sc, sh, eps=1e-6)
    ref = _ln64(syn.bf16_bits_to_f32(bits).astype(np.float64), syn.bf16_bits_to_f32(sc).astype(np.float64),
                syn.bf16_bits_to_f32(sh).astype(np.float64), 1e-6)
    assert np.abs(m - ref).max() <= 2e-5 * (np.abs(ref).max() + 1)
    # without the modulation vectors it is the plain LayerNorm
    m0 = oracle.ln_modulate(bits, None, None, eps=1e-6)
    ref0 = _ln64(syn.bf16_bits_to_f32(bits).astype(np.float64), 0.0, 0.0, 1e-6)
    assert np.abs(m0 - ref0).max() <= 2e-5 * (np.abs(ref0).max() + 1)


def test_constant_row_gives_the_shift_exactly():
    x = np.full((2, 64), 0x3FC0, np.uint16)  # 1.5
    sh = syn.normal_bf16((64,), seed=3)
    m = oracle.ln_modulate(x, syn.normal_bf16((64,), seed=4), sh)
    assert np.array_equal(m, np.broadcast_to(syn.bf16_bits_to_f32(sh), (2, 64)))


def test_population_variance_and_eps_inside_the_root():
    # +-2 alternating: mean 0, population variance 4 (a sample variance would be 4 * 64/63)
    x = np.tile(np.array([0x4000, 0xC000], np.uint16), (1, 32))  # 2, -2
    eps = 0.25
    m = oracle.ln_modulate(x, None, None, eps=eps)
    want = np.float32(2.0) / np.sqrt(np.float32(4.0 + eps))
    assert np.allclose(np.abs(m), want, rtol=1e-6, atol=0)
    assert np.all(np.sign(m[0, 0::2]) > 0) and np.all(np.sign(m[0, 1::2]) < 0)


def test_quantize_of_the_modulated_rows_is_the_binary32_quantize():
    bits = syn.activations_bf16(32, 256, seed=8)
    codes, scales, a32 = oracle.ln_modulate_quantize(bits, syn.normal_bf16((256,), seed=9, std=0.1), None)
    m = oracle.ln_modulate(bits, syn.normal_bf16((256,), seed=9, std=0.1), None)
    assert a32 == np.float32(np.abs(m).max() / np.float32(2688.0))
    c2, s2, a2 = oracle.quantize(m)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2) and a2 == a32


def _f32_round(q: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) binary32 of the rational q."""
    f = np.float32(float(q))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        key = (abs(Fraction(float(c)) - q), int(np.array(c, np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


@pytest.mark.parametrize("rows,cols", [(6, 3072), (4, 64), (3, 1040)])
def test_row_mean_is_the_correctly_rounded_exact_mean(rows, cols):
    # the mean statistic is fl32 of the exact rational mean (bf16 sums are exact in binary64 here)
    bits = syn.activations_bf16(rows, cols, seed=3 * rows + cols)
    st = oracle.ln_stats(bits, eps=1e-6)
    x = syn.bf16_bits_to_f32(bits)
    for r in range(rows):
        mu = sum(Fraction(float(v)) for v in x[r]) / cols
        assert st[r, 0] == _f32_round(mu), r


@pytest.mark.parametrize("rows,cols", [(6, 3072), (4, 64)])
def test_row_rstd_is_within_one_unit_of_the_exact_value(rows, cols):
    # rstd = 1 / sqrt(var + eps) with the exact population variance: the binary64 route is within one
    # binary32 unit of it (a block left out, n - 1, or squares about 0 move it by far more)
    bits = syn.activations_bf16(rows, cols, seed=5 * rows + cols)
    eps = 1e-6
    st = oracle.ln_stats(bits, eps=eps)
    x = syn.bf16_bits_to_f32(bits)
    for r in range(rows):
        xs = [Fraction(float(v)) for v in x[r]]
        mu = sum(xs) / cols
        var = sum((v - mu) ** 2 for v in xs) / cols
        want = 1.0 / np.sqrt(float(var + Fraction(eps)))
        got = float(st[r, 1])
        assert abs(got - want) <= float(np.spacing(np.float32(want))), r


def test_modulation_given_statistics_is_the_binary32_expression():
    # with (mean, rstd) given, every element is fl32(fl32(fl32(fl32(x - mean) rstd) fl32(1 + sc)) + sh),
    # restated here with numpy binary32 operations (each correctly rounded, no fusion)
    rows, cols = 5, 320
    bits = syn.activations_bf16(rows, cols, seed=21)
    sc = syn.normal_bf16((cols,), seed=22, std=0.1)
    sh = syn.normal_bf16((cols,), seed=23, std=0.1)
    rng = np.random.default_rng(24)
    st = np.stack([rng.standard_normal(rows), rng.uniform(0.5, 2.0, rows)], axis=1).astype(np.float32)
    m = oracle.ln_modulate(bits, sc, sh, stats=st)
    x = syn.bf16_bits_to_f32(bits)
    f = np.float32
    h = (x - st[:, :1].astype(f)).astype(f) * st[:, 1:].astype(f)
    g = (f(1.0) + syn.bf16_bits_to_f32(sc)).astype(f)
    want = (h.astype(f) * g).astype(f) + syn.bf16_bits_to_f32(sh)
    assert np.array_equal(m, want.astype(f))
    # and the quantize of it is the binary32 quantize of m
    c1, s1, a1 = oracle.ln_modulate_quantize(bits, sc, sh, stats=st)
    c2, s2, a2 = oracle.quantize(m)
    assert np.array_equal(c1, c2) and np.array_equal(s1, s2) and a1 == a2
