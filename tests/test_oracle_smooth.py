"""Pins of the oracle's K-smoothing (R20) against exact arithmetic and closed forms.

Source: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (reading note), section 二,
推理底座, second item: each frame-chunk's K and V get K-smoothing and an
adaptive scale before the NVFP4 store.  The pages name the step only; the
reading (channel mean over the chunk's tokens, subtracted before the
quantize, added back in the dequant, binary32 in a fixed order) is R20.
"""
from fractions import Fraction

import numpy as np
import pytest

import oracle

pytestmark = pytest.mark.filterwarnings("ignore::RuntimeWarning")


def bf16_bits(f32: np.ndarray) -> np.ndarray:
    """binary32 values that are exact in bf16 -> their bf16 bit patterns."""
    b = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32)
    assert np.all((b & 0xFFFF) == 0), "value not exact in bf16"
    return (b >> 16).astype(np.uint16)


def bf16_value(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def bf16_rne(f32: np.ndarray) -> np.ndarray:
    """Textbook binary32 -> bf16 nearest-even on the bit pattern (finite inputs)."""
    b = np.ascontiguousarray(f32, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def f32_round(q: Fraction) -> np.float32:
    """Correctly rounded (nearest, ties to even) binary32 of the rational q."""
    f = np.float32(float(q))
    best = None
    for c in (np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))):
        d = abs(Fraction(float(c)) - q)
        key = (d, int(np.array(c, np.float32).view(np.uint32)) & 1)
        if best is None or key < best[0]:
            best = (key, c)
    return np.float32(best[1])


def grid_values(rng, shape, lim=8.0):
    """Multiples of 1/8 in [-lim, lim]: every partial and total sum below is exact in binary32."""
    return (rng.integers(-int(lim * 8), int(lim * 8) + 1, size=shape) / 8.0).astype(np.float32)


def test_channel_mean_is_the_correctly_rounded_mean_when_sums_are_exact():
    # 2640 tokens (the chunk length of the KV workload) x 48 channels; all sums are exact,
    # so the only rounding is the final division, whatever the order
    rng = np.random.default_rng(11)
    T, C = 2640, 48
    x = grid_values(rng, (T, C))
    m = oracle.channel_mean(bf16_bits(x))
    for c in range(C):
        S = sum(Fraction(float(v)) for v in x[:, c])
        assert m[c] == f32_round(S / T), c


def test_channel_mean_of_a_constant_channel_is_that_constant():
    rng = np.random.default_rng(12)
    T, C = 2640, 64
    b = grid_values(rng, (C,))
    x = np.broadcast_to(b, (T, C)).copy()
    assert np.array_equal(oracle.channel_mean(bf16_bits(x)), b)


@pytest.mark.parametrize("T", [1, 31, 33, 100, 2640])
def test_channel_mean_is_the_correctly_rounded_exact_mean(T):
    # R20 is the definition: fl32 of the exact mean, whatever the data (a token dropped or counted
    # twice, or a wrong channel stride, moves it by ~|x| / T)
    rng = np.random.default_rng(T)
    C = 3 * 32
    x = bf16_value(bf16_rne(rng.standard_normal((T, C)).astype(np.float32)))
    m = oracle.channel_mean(bf16_bits(x))
    for c in range(C):
        assert m[c] == f32_round(sum(Fraction(float(v)) for v in x[:, c]) / T), c


def summation_bound(x: np.ndarray, mean: np.ndarray) -> np.ndarray:
    """Bound on |m - mean| for binary32 channel means m summed as 32 strided
    partial sums (each over ceil(T/32) tokens in order) met in 5 pairwise
    levels, then divided by T: every term passes through at most
    ceil(T/32) + 5 rounded additions, and the division adds one rounding."""
    T = x.shape[0]
    u = 2.0 ** -24
    depth = -(-T // 32) + 5
    return (depth + 1) * u * np.abs(x.astype(np.float64)).sum(0) / T + u * np.abs(mean)


@pytest.mark.parametrize("T", [1, 33, 2640])
def test_summation_bound_holds_for_strided_partials_and_catches_a_dropped_token(T):
    # The GPU tests hold a kernel's channel means to summation_bound.  A binary32 sum in that
    # shape (32 strided partials, pairwise levels) stays inside it; the same sum with one
    # token left out does not.
    rng = np.random.default_rng(100 + T)
    C = 64
    x = bf16_value(bf16_rne((rng.standard_normal((T, C)) + 3.0).astype(np.float32)))
    mean = oracle.channel_mean(bf16_bits(x)).astype(np.float64)
    bound = summation_bound(x, mean)

    def strided(xs):
        part = np.zeros((32, C), np.float32)
        for t in range(xs.shape[0]):
            part[t % 32] = (part[t % 32] + xs[t]).astype(np.float32)
        while part.shape[0] > 1:
            h = part.shape[0] // 2
            part = (part[:h] + part[h:]).astype(np.float32)
        return (part[0] / np.float32(T)).astype(np.float32).astype(np.float64)

    assert np.all(np.abs(strided(x) - mean) <= bound)
    if T > 1:
        short = strided(np.delete(x, T // 2, axis=0))
        assert np.all(np.abs(short - mean) > bound)


def test_channel_constant_chunk_round_trips_exactly_with_smoothing_only():
    # K[t, h, j] = b[h, j]: smoothing leaves all-zero values, so the chunk's tensor scale is 0
    # (R2), every code and scale is 0, and the dequant returns the mean, which is b exactly
    rng = np.random.default_rng(13)
    T, H, d = 96, 3, 32
    b = grid_values(rng, (H, d), lim=4.0)
    b[0, 0] = 3.375  # at least one value off the {4,6}-friendly grid of one block
    x = np.broadcast_to(b, (T, H, d)).copy()
    xb = bf16_bits(x)
    codes, scales, alpha, mean = oracle.kv_append_smooth(xb)
    assert alpha == 0.0
    assert not codes.any() and not scales.any()
    assert np.array_equal(mean, b.reshape(-1))
    assert np.array_equal(oracle.kv_dequant_smooth(codes, scales, alpha, mean, T, H, d), xb)
    # the plain store does not reproduce this chunk (the test has teeth)
    c2, s2, a2 = oracle.kv_append(xb)
    assert not np.array_equal(oracle.kv_dequant(c2, s2, a2, T, H, d), xb)


@pytest.mark.parametrize("search46", [False, True])
def test_smoothed_store_is_the_plain_store_of_the_centred_chunk(search46):
    # x = b + z with z[t + 32] = -z[t] over 64 tokens: every partial sum is (b + z) + (b - z) = 2b
    # exactly, so the mean is b exactly and x - mean = z exactly.  The smoothed store of x is then
    # the plain store of z, and its dequant is bf16(fl32(dequant_f32(z) + b)).
    rng = np.random.default_rng(14 + search46)
    T, H, d = 64, 4, 32
    b = grid_values(rng, (H, d), lim=8.0)
    z = grid_values(rng, (32, H, d), lim=7.0)
    z = np.concatenate([z, -z], axis=0) + np.float32(0.0)  # -0.0 -> +0.0, as x - mean gives
    x = (b[None] + z).astype(np.float32)
    codes, scales, alpha, mean = oracle.kv_append_smooth(bf16_bits(x), search46=search46)
    assert np.array_equal(mean, b.reshape(-1))
    pc, ps, pa = oracle.kv_append(bf16_bits(z), search46=search46)
    assert alpha == pa
    assert np.array_equal(codes, pc) and np.array_equal(scales, ps)
    got = oracle.kv_dequant_smooth(codes, scales, alpha, mean, T, H, d)
    dq = oracle.dequant_f32(pc, ps, pa).reshape(T, H, d)
    want = bf16_rne((dq + b[None]).astype(np.float32))
    assert np.array_equal(got, want)
    # and the mean really was added: without it the result differs
    assert not np.array_equal(got, oracle.kv_dequant(pc, ps, pa, T, H, d))
