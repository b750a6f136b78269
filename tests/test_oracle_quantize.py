"""Pins of the oracle's NVFP4 quantize / dequant / scale layout.

What pins them (none of it re-types the oracle's own steps):
- the three-level scaling and the Dequant equation of "LongLive-2.0：用 NVFP4
  并行底座做长视频生成" (yingwang.github.io reading note), section 二 方法 /
  "NVFP4 量化格式": every element's code must be the nearest grid point of
  x / (s * a32) (checked in exact rational arithmetic with a one-binary32-ulp
  slack for the reciprocal), which fails on a wrong scale, sign, rounding,
  block boundary or nibble order;
- invariants: the block amax maps to code +-6 whenever the block scale is a
  normal E4M3 number; the block holding the tensor amax gets scale 448 (the
  6*448 tensor scale, R1); re-quantizing a dequantized tensor with the same
  tensor scale returns the same codes;
- the zero / flushed / subnormal-scale special cases (R2, R4);
- a hand-worked table of scale-tile offsets and the bijectivity of the layout.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from bit_video_dit_b200 import synthetic as syn

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def _codes_unpacked(codes: np.ndarray) -> np.ndarray:
    lo = codes & 0xF
    hi = codes >> 4
    return np.stack([lo, hi], axis=-1).reshape(codes.shape[0], -1)


def _grid_value(code: int) -> float:
    v = GRID[code & 7]
    return -v if code & 8 else v


def test_quantize_codes_are_nearest_grid_points():
    x = syn.tiny_a_bf16(32, 128, seed=21)
    codes, scales, a32 = oracle.quantize(x)
    xf = syn.bf16_bits_to_f32(x)
    q = _codes_unpacked(codes)
    for r in range(x.shape[0]):
        for b in range(x.shape[1] // 16):
            s = oracle.e4m3_value(int(scales[r, b]))
            if s == 0.0:
                assert (q[r, 16 * b:16 * b + 16] == 0).all()
                continue
            denom = Fraction(float(np.float32(s) * np.float32(a32)))
            for i in range(16 * b, 16 * b + 16):
                y = Fraction(float(xf[r, i])) / denom
                got = Fraction(_grid_value(int(q[r, i])))
                if abs(y) >= 6:
                    assert abs(got) == 6
                    continue
                best = min(abs(abs(y) - Fraction(g)) for g in GRID)
                slack = abs(y) * Fraction(1, 2 ** 22)
                assert abs(abs(y) - abs(got)) <= best + slack, (r, i, float(y), float(got))
                if got != 0:
                    assert (got < 0) == (y < 0)


def test_block_amax_maps_to_six_for_normal_scales():
    x = syn.activations_bf16(64, 512, seed=3)
    codes, scales, _ = oracle.quantize(x)
    xf = np.abs(syn.bf16_bits_to_f32(x))
    q = _codes_unpacked(codes) & 7
    checked = 0
    for r in range(64):
        for b in range(512 // 16):
            if scales[r, b] >= 0x08:  # normal E4M3 block scale
                i = 16 * b + int(np.argmax(xf[r, 16 * b:16 * b + 16]))
                assert q[r, i] == 7
                checked += 1
    assert checked > 1000


def test_tensor_amax_block_gets_scale_448():
    for seed in range(5):
        x = syn.activations_bf16(48, 256, seed=seed)
        codes, scales, a32 = oracle.quantize(x)
        xf = np.abs(syn.bf16_bits_to_f32(x))
        r, c = np.unravel_index(int(np.argmax(xf)), xf.shape)
        assert scales[r, c // 16] == 0x7E
        assert a32 == np.float32(np.float32(xf.max()) / np.float32(2688.0))


def test_all_zero_tensor():
    x = np.zeros((16, 64), np.uint16)
    codes, scales, a32 = oracle.quantize(x)
    assert a32 == 0.0 and not codes.any() and not scales.any()


def test_all_zero_block_and_flushed_block():
    xf = np.random.default_rng(1).standard_normal((4, 64)).astype(np.float32)
    xf[1, 16:32] = 0.0
    xf[2, 32:48] = np.float32(1e-6) * np.sign(xf[2, 32:48])  # r_b far below 2^-10 -> flushed (R4)
    x = syn.f32_to_bf16_bits(xf)
    codes, scales, a32 = oracle.quantize(x)
    q = _codes_unpacked(codes)
    assert scales[1, 1] == 0 and not q[1, 16:32].any()
    assert scales[2, 2] == 0 and not q[2, 32:48].any()


def test_negative_values_rounding_to_zero_keep_sign():
    xf = np.zeros((1, 16), np.float32)
    xf[0, 0] = 6.0
    xf[0, 1] = -0.1   # |y| = 0.1 -> rounds to zero, code 0x8 (R7)
    xf[0, 2] = 0.1
    codes, scales, _ = oracle.quantize(syn.f32_to_bf16_bits(xf), alpha=np.float32(1.0 / 64))
    q = _codes_unpacked(codes)[0]
    assert q[0] == 7 and q[1] == 8 and q[2] == 0


def test_subnormal_scale_band_error_bound():
    # r_b = amax_b / (6 a32) in the E4M3 subnormal band [2^-9, 2^-6): the
    # scale is coarse, the amax->6 invariant may fail, but every element
    # still sits within half a grid step of x / (s a32).
    a32 = np.float32(1.0)
    xf = np.random.default_rng(2).uniform(-1, 1, (8, 64)).astype(np.float32)
    xf *= np.float32(6 * 2.0 ** -8)
    codes, scales, _ = oracle.quantize(syn.f32_to_bf16_bits(xf), alpha=a32)
    assert (scales < 0x08).all() and (scales > 0).any()
    x2 = syn.bf16_bits_to_f32(syn.f32_to_bf16_bits(xf))
    dq = oracle.dequant_f32(codes, scales, a32)
    for r in range(8):
        for b in range(4):
            s = oracle.e4m3_value(int(scales[r, b]))
            blk = slice(16 * b, 16 * b + 16)
            ratio = np.abs(x2[r, blk]) / s
            err = np.abs(x2[r, blk] - dq[r, blk]) / s
            # half the E2M1 gap at that magnitude, or saturation past 6
            half_gap = np.where(ratio < 2, 0.25, np.where(ratio < 4, 0.5, 1.0))
            ok = (err <= half_gap * (1 + 1e-6)) | (ratio > 6)
            assert ok.all()


def test_requantize_dequantized_is_identity():
    x = syn.activations_bf16(32, 256, seed=9)
    codes, scales, a32 = oracle.quantize(x)
    dq = oracle.dequant_f32(codes, scales, a32)
    q = _codes_unpacked(codes) & 7
    c2, s2, a2 = oracle.quantize(dq, alpha=a32)
    assert a2 == a32
    # blocks whose max code is 6 and scale is normal reproduce exactly
    for r in range(32):
        for b in range(256 // 16):
            if scales[r, b] >= 0x08 and q[r, 16 * b:16 * b + 16].max() == 7:
                assert s2[r, b] == scales[r, b]
                assert (c2[r, 8 * b:8 * b + 8] == codes[r, 8 * b:8 * b + 8]).all()


def test_dequant_equation_closed_form():
    # Dequant(X) = X^FP4 * a^FP8 * a^FP32 for hand-picked codes
    codes = np.array([[0x71, 0xF8] + [0] * 6], np.uint8)  # elements: 0.5, 6, -0, -6, zeros
    scales = np.array([[0x38]], np.uint8)                 # E4M3 0x38 = 1.0
    a32 = np.float32(0.25)
    out = oracle.dequant_f32(codes, scales, a32)[0]
    assert list(out[:4]) == [0.125, 1.5, 0.0, -1.5]
    assert np.signbit(out[2])
    scales2 = np.array([[0x48]], np.uint8)                # E4M3 0x48 = 4.0
    out2 = oracle.dequant_f32(codes, scales2, a32)[0]
    assert list(out2[:4]) == [0.5, 6.0, 0.0, -6.0]


def test_swizzle_golden_offsets(golden):
    for rows, sc, r, c, off in golden("swizzle_offsets.txt"):
        assert oracle.swizzle_offset(int(r), int(c), int(sc)) == int(off), (rows, sc, r, c)


@pytest.mark.parametrize("rows,sc", [(128, 4), (256, 8), (200, 12), (1, 4), (300, 192)])
def test_swizzle_is_a_bijection_with_zero_padding(rows, sc):
    g = np.random.default_rng(rows * 1000 + sc)
    logical = g.integers(1, 255, size=(rows, sc), dtype=np.uint8)
    swz = oracle.swizzle(logical)
    assert swz.size == ((rows + 127) // 128) * 128 * ((sc + 3) // 4) * 4
    assert (oracle.unswizzle(swz, rows, sc) == logical).all()
    assert np.count_nonzero(swz) == rows * sc  # padding bytes stay zero
    offs = {oracle.swizzle_offset(r, c, sc) for r in range(0, rows, 7) for c in range(sc)}
    assert len(offs) == len(range(0, rows, 7)) * sc


def test_reciprocal_form_decides_a_midpoint():
    """R5: the element is multiplied by the binary32 reciprocal of s * a32, not divided by it.  With a32 = 1
    (given) and a block max of 0.17578125 the block scale is s = 0.029296875 (E4M3 1.875 * 2^-6) exactly, and
    the element 0.0732421875 = 2.5 * s sits on the E2M1 midpoint between 2 and 3: divided by s it is 2.5 and
    ties to 2 (code 4); times fl32(1 / s) it is 2.5000002 and rounds to 3 (code 5).  The expected codes come
    from numpy binary32 arithmetic and ml_dtypes' E4M3 / E2M1 conversions (round to nearest even)."""
    import ml_dtypes

    xf = np.zeros((1, 16), np.float32)
    xf[0, 0], xf[0, 1] = 0.17578125, 0.0732421875
    codes, scales, _ = oracle.quantize(xf, alpha=np.float32(1.0))
    r = np.array([np.float32(0.17578125) / np.float32(6.0)], np.float32)
    s = r.astype(ml_dtypes.float8_e4m3fn).astype(np.float32)[0]
    assert s == np.float32(0.029296875) and scales[0, 0] == r.astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
    inv = np.float32(1.0) / (s * np.float32(1.0))
    want = (np.minimum(xf[0] * inv, np.float32(6.0)).astype(ml_dtypes.float4_e2m1fn).view(np.uint8) & 0xF).tolist()
    q = _codes_unpacked(codes)[0].tolist()
    assert q == want and q[1] == 5
    # the division form would have given code 4 for that element
    yd = np.array([xf[0, 1] / s], np.float32)
    assert int(yd.astype(ml_dtypes.float4_e2m1fn).view(np.uint8)[0] & 0xF) == 4


def test_dequant_rounds_to_binary32_then_to_bf16():
    """R10: two roundings, binary32 then bf16.  With sixteen elements of 1.5, scale 1 and a32 = 0.66927087307
    (binary32), the exact product 1.5 * a32 = 1.0039063096... rounds in binary32 to 1 + 2^-8, the midpoint
    between the bf16 values 1 and 1 + 2^-7, which ties to 1 (bf16 0x3F80); one rounding of the exact product
    would give 1 + 2^-7 (0x3F81).  The expected value is torch's binary32 -> bf16 conversion of numpy's
    binary32 product."""
    import torch

    a32 = np.float32(0.6692708730697632)
    codes = np.full((1, 8), 0x33, np.uint8)  # elements 1.5 (code 3) in both nibbles
    scales = np.array([[0x38]], np.uint8)    # E4M3 0x38 = 1.0
    got = oracle.dequant_bf16(codes, scales, a32)[0]
    p32 = np.float32(1.5) * a32
    want = torch.tensor([p32]).to(torch.bfloat16).view(torch.int16).item() & 0xFFFF
    assert p32 == np.float32(1.0 + 2.0 ** -8) and want == 0x3F80
    assert all(int(v) == want for v in got)
    # the exact product lies above the midpoint, so a single rounding would go up
    assert Fraction(3, 2) * Fraction(float(a32)) > Fraction(1) + Fraction(1, 256)
