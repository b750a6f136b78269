"""Pins of the oracle's LayerNorm + adaLN modulate before the quantize
(reading R19: population variance, eps inside the square root, no affine
LayerNorm parameters, m = h * (1 + scale) + shift), against a float64 numpy
LayerNorm and closed-form rows."""
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
