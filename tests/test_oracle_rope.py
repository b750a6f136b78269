"""Pins of the oracle's rotary position embedding of KV keys (reading R24:
interleaved pairs (2p, 2p+1) of every head turned by the (token, p) angle of a
binary32 cos/sin table, y0 = fl32(fl32(x0 c) - fl32(x1 s)), y1 = fl32(fl32(x0 s)
+ fl32(x1 c)), ahead of the keys' quantize; with K-smoothing the means are taken
over the rotated keys).  The fused RoPE ahead of the in-place KV update is the
anzhuoshouzhuan.com LongLive 2.0 article's "NVFP4 量化" section.

Each pin is fixed by the mathematics, not by retyping the oracle: the complex
product in fp64 with a rounding bound, turns by 0, a quarter and a half (exact
in binary32), an index pin on one pair of one token, and the append path against
the already-pinned plain and smoothed appends on exactly transformed inputs."""
import numpy as np
import pytest

import oracle
from bit_video_dit_b200 import synthetic as syn

U = 2.0 ** -24


def _f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def _nonzero_chunk(T, H, d, seed):
    """A seeded K chunk with no zero elements (so the sign of a zero never decides a code)."""
    k, _ = syn.kv_chunk_bf16(T, H, d, seed=seed)
    k = k.copy()
    k[(k & 0x7FFF) == 0] = 0x3C00  # 2^-7
    return k


def _turn(T, d, c, s):
    return np.full((T, d // 2), c, np.float32), np.full((T, d // 2), s, np.float32)


def test_complex_product_within_three_roundings():
    T, H, d = 24, 3, 32
    x = _nonzero_chunk(T, H, d, seed=1)
    cs, sn = syn.rope_table(T, d, seed=2)
    y = oracle.rope(x, cs, sn).astype(np.float64)
    xf = _f32(x).astype(np.float64).reshape(T, H, d // 2, 2)
    z = (xf[..., 0] + 1j * xf[..., 1]) * (cs.astype(np.float64) + 1j * sn.astype(np.float64))[:, None, :]
    ref = np.stack([z.real, z.imag], axis=-1).reshape(T, H, d)
    # |c|, |s| <= 1: two rounded products and a rounded sum, each relative U
    bound = 2.02 * U * (np.abs(xf[..., 0]) + np.abs(xf[..., 1]))
    bound = np.repeat(bound, 2, axis=-1).reshape(T, H, d)
    assert np.all(np.abs(y - ref) <= bound)
    # and it is not the identity: the angles do move the values
    assert np.max(np.abs(y - _f32(x))) > 0.5


def test_zero_quarter_and_half_turns_are_exact():
    T, H, d = 8, 2, 16
    x = _nonzero_chunk(T, H, d, seed=3)
    xf = _f32(x)
    assert np.array_equal(oracle.rope(x, *_turn(T, d, 1.0, 0.0)), xf)
    q = oracle.rope(x, *_turn(T, d, 0.0, 1.0))
    assert np.array_equal(q[..., 0::2], -xf[..., 1::2]) and np.array_equal(q[..., 1::2], xf[..., 0::2])
    h = oracle.rope(x, *_turn(T, d, -1.0, 0.0))
    assert np.array_equal(h, -xf)


def test_one_pair_of_one_token_turns_in_every_head():
    """Only token 5's pair 3 gets a quarter turn: exactly channels 6 and 7 of that
    token change, in every head (table rows are tokens, columns pairs)."""
    T, H, d = 9, 4, 16
    x = _nonzero_chunk(T, H, d, seed=4)
    cs, sn = _turn(T, d, 1.0, 0.0)
    cs[5, 3], sn[5, 3] = 0.0, 1.0
    y = oracle.rope(x, cs, sn)
    xf = _f32(x)
    changed = np.argwhere(y != xf)
    assert {(int(t), int(j)) for t, _, j in changed} == {(5, 6), (5, 7)}
    assert len(changed) == 2 * H
    assert np.array_equal(y[5, :, 6], -xf[5, :, 7]) and np.array_equal(y[5, :, 7], xf[5, :, 6])


def _quarter_turned_bits(x):
    """bf16 bits of the exact quarter turn: (x0, x1) -> (-x1, x0)."""
    y = x.copy()
    y[..., 0::2] = x[..., 1::2] ^ 0x8000
    y[..., 1::2] = x[..., 0::2]
    return y


@pytest.mark.parametrize("search46", [False, True])
def test_append_equals_the_plain_append_of_the_turned_keys(search46):
    T, H, d = 12, 3, 32
    x = _nonzero_chunk(T, H, d, seed=5)
    got = oracle.kv_append_rope(x, *_turn(T, d, 0.0, 1.0), search46=search46)
    ref = oracle.kv_append(_quarter_turned_bits(x), search46=search46)
    assert np.array_equal(got[0], ref[0]) and np.array_equal(got[1], ref[1]) and got[2] == ref[2]
    assert got[3] is None
    ident = oracle.kv_append_rope(x, *_turn(T, d, 1.0, 0.0), search46=search46)
    plain = oracle.kv_append(x, search46=search46)
    assert all(np.array_equal(a, b) for a, b in zip(ident[:3], plain[:3]))


def test_smoothed_append_takes_the_means_of_the_rotated_keys():
    T, H, d = 70, 2, 16
    x = _nonzero_chunk(T, H, d, seed=6)
    got = oracle.kv_append_rope(x, *_turn(T, d, 0.0, 1.0), smooth=True)
    ref = oracle.kv_append_smooth(_quarter_turned_bits(x))
    for a, b in zip(got, ref):
        assert np.array_equal(a, b)
    # the quarter turn negates and swaps channels, and so do the means, exactly
    m = oracle.channel_mean(x)
    assert np.array_equal(got[3][0::2], -m[1::2]) and np.array_equal(got[3][1::2], m[0::2])


def test_channel_mean_f32_matches_the_bf16_order_and_a_constant_angle_commutes():
    T, H, d = 75, 2, 32
    x = _nonzero_chunk(T, H, d, seed=7)
    assert np.array_equal(oracle.channel_mean_f32(_f32(x)), oracle.channel_mean(x))
    # one angle for all tokens: the mean of the rotated keys is the rotated mean
    # (linear map), up to the roundings of T additions and of the rotation
    cs, sn = _turn(T, d, np.float32(np.cos(0.7)), np.float32(np.sin(0.7)))
    my = oracle.channel_mean_f32(oracle.rope(x, cs, sn)).astype(np.float64).reshape(H, d // 2, 2)
    mx = oracle.channel_mean(x).astype(np.float64).reshape(H, d // 2, 2)
    c, s = float(cs[0, 0]), float(sn[0, 0])
    r0 = mx[..., 0] * c - mx[..., 1] * s
    r1 = mx[..., 0] * s + mx[..., 1] * c
    scale = np.abs(_f32(x)).max()
    assert np.max(np.abs(my[..., 0] - r0)) <= 4 * T * U * scale
    assert np.max(np.abs(my[..., 1] - r1)) <= 4 * T * U * scale


def test_tables_are_checked():
    x = _nonzero_chunk(4, 1, 16, seed=8)
    with pytest.raises(ValueError):
        oracle.rope(x, np.ones((4, 7), np.float32), np.zeros((4, 7), np.float32))


def test_workload_table_shape_and_unit_norm():
    cs, sn = syn.rope_table_3d(*syn.KV_GRID, syn.KV_DIM)
    assert cs.shape == (syn.KV_TOKENS, syn.KV_DIM // 2)
    n = cs.astype(np.float64) ** 2 + sn.astype(np.float64) ** 2
    assert np.max(np.abs(n - 1.0)) < 4 * U
    # frame band: pairs 0..21 depend only on the frame index (880 tokens per frame)
    assert np.array_equal(cs[0, :22], cs[879, :22]) and not np.array_equal(cs[0, :22], cs[880, :22])
