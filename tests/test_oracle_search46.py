"""Pins of the oracle's adaptive scale search over the targets {4, 6} (reading
R18 of the pages' "adaptive scale search" with the magnitude targets {4, 6}):
per 16-element block the encoding with the block max aimed at 4 replaces the
standard one (aimed at 6) when its squared error is smaller.

Checked against things outside the oracle: hand-built blocks that one of the
two targets represents exactly, ml_dtypes decodes of the codes and scales, and
the E4M3 rounding of amax_b / (4 a32) done by ml_dtypes."""
import ml_dtypes
import numpy as np
import pytest

import oracle
from bit_video_dit_b200 import synthetic as syn

E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6], np.float64)


def _decode(codes, scales, alpha):
    """float64 dequant from the raw codes and scales (ml_dtypes for E4M3)."""
    R = codes.shape[0]
    lo = codes & 0xF
    hi = codes >> 4
    q = np.empty((R, codes.shape[1] * 2), np.uint8)
    q[:, 0::2] = lo
    q[:, 1::2] = hi
    s = scales.view(ml_dtypes.float8_e4m3fn).astype(np.float64)
    return E2M1[q] * np.repeat(s, 16, axis=1) * np.float64(alpha), s


def _block(vals):
    x = np.zeros((1, 16), np.float32)
    x[0, :len(vals)] = vals
    return x


def test_block_exact_under_target_4_takes_it():
    # a32 = 1: aimed at 4 the scale is exactly 1.0 and every element is on the grid;
    # aimed at 6 the scale is E4M3(4/6) = 0.6875 and 4 no longer decodes exactly
    x = _block([4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 4, 2, 1])
    c6, s6, _ = oracle.quantize(x, alpha=1.0)
    c46, s46, _ = oracle.quantize(x, alpha=1.0, search46=True)
    assert s6[0, 0] == 0x33  # 0.6875 = 1.375 * 2^-1
    assert s46[0, 0] == 0x38  # 1.0
    deq, _ = _decode(c46, s46, 1.0)
    assert np.array_equal(deq[0], x[0].astype(np.float64))
    deq6, _ = _decode(c6, s6, 1.0)
    assert np.abs(deq6[0] - x[0]).max() > 0


def test_block_exact_under_target_6_keeps_it():
    x = _block([6, 3, 1.5, 0.5, 0, -6, 2, 1, -0.5, 4, -3, 1.5, 0, 0, 6, -1])
    c6, s6, _ = oracle.quantize(x, alpha=1.0)
    c46, s46, _ = oracle.quantize(x, alpha=1.0, search46=True)
    assert np.array_equal(c46, c6) and np.array_equal(s46, s6)
    deq, _ = _decode(c46, s46, 1.0)
    assert np.array_equal(deq[0], x[0].astype(np.float64))


def test_a_tie_keeps_the_standard_encoding():
    """Sixteen 6.0 with a32 = 1 are exact under both targets: aimed at 6 the scale is 1.0 and every code
    is 6; aimed at 4 the scale is 1.5 and every code is 4.  Both squared errors are 0, and a tie keeps the
    standard encoding (scale E4M3 0x38 = 1.0, not 0x3C = 1.5)."""
    x = _block([6.0] * 16)
    c46, s46, _ = oracle.quantize(x, alpha=1.0, search46=True)
    one = np.array([1.0], np.float32).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)[0]
    assert s46[0, 0] == one == 0x38
    deq, _ = _decode(c46, s46, 1.0)
    assert np.array_equal(deq[0], x[0].astype(np.float64))
    # the target-4 candidate is exact too: its scale 6 / 4 = 1.5 is an E4M3 value
    assert np.array([1.5], np.float32).astype(ml_dtypes.float8_e4m3fn).astype(np.float32)[0] == 1.5


def test_zero_tensor_and_flushed_blocks_unchanged():
    x = np.zeros((3, 64), np.float32)
    assert all(np.array_equal(a, b) for a, b in zip(oracle.quantize(x)[:2], oracle.quantize(x, search46=True)[:2]))
    x[1, 17] = 1e-30  # flushed block beside zero blocks
    x[2, :] = 1.0
    r0, r1 = oracle.quantize(x), oracle.quantize(x, search46=True)
    assert np.array_equal(r0[0][:2], r1[0][:2]) and np.array_equal(r0[1][:2], r1[1][:2])


@pytest.mark.parametrize("seed", [3, 4])
def test_random_blocks_search_never_worse_and_uses_target_4_scale(seed):
    bits = syn.activations_bf16(64, 1024, seed=seed)
    x = syn.bf16_bits_to_f32(bits)
    c6, s6, a6 = oracle.quantize(bits)
    c46, s46, a46 = oracle.quantize(bits, search46=True)
    assert a6 == a46  # the tensor scale is R1's
    d6, _ = _decode(c6, s6, a6)
    d46, _ = _decode(c46, s46, a46)
    xb = x.astype(np.float64).reshape(64, -1, 16)
    e6 = ((d6.reshape(64, -1, 16) - xb) ** 2).sum(-1)
    e46 = ((d46.reshape(64, -1, 16) - xb) ** 2).sum(-1)
    scale = np.maximum(e6, 1e-300)
    assert np.all(e46 <= e6 * (1 + 1e-5) + 1e-30)
    changed = s46 != s6
    assert changed.any() and (~changed).any()
    # where the search switched, it did so for a clearly better encoding, and the new
    # scale is E4M3 nearest-even (ml_dtypes) of amax_b / fl32(4 a32)
    assert np.all(e46[changed] < e6[changed] * (1 + 1e-5))
    amax_b = np.abs(x.reshape(64, -1, 16)).max(-1)
    d4 = np.float32(4.0) * np.float32(a6)
    r4 = (amax_b / d4).astype(np.float32)
    want = np.minimum(r4, np.float32(448)).astype(ml_dtypes.float8_e4m3fn).view(np.uint8)
    assert np.array_equal(s46[changed], want[changed])
    # scales and codes elsewhere stay the standard ones
    assert np.array_equal(s46[~changed], s6[~changed])


def test_kv_append_search_matches_quantize_search():
    k, _ = syn.kv_chunk_bf16(64, 4, 128, seed=9)
    codes, scales, a = oracle.kv_append(k, search46=True)
    c2, s2, a2 = oracle.quantize(k.reshape(64 * 4, 128), search46=True)
    assert np.array_equal(codes, c2) and np.array_equal(scales, s2) and a == a2
