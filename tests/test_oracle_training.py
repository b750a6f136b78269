"""Pins of the oracle's training-side NVFP4 operands: 2D block scaling of
weights (R21) and the transposed quantize with the 16-point Random Hadamard
Transform ahead of the weight-gradient GEMM (R22).

Source: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (reading note), section
"NVFP4 训练的工程细节": weights use 2D block scaling (blocks along both
dimensions), activations and gradients 1D block scaling, and a Random Hadamard
Transform precedes the quantize of the weight-gradient GEMM's inputs.

What pins them (none of it re-types the oracle's steps): the Sylvester Hadamard
matrix of scipy on exact inputs; the 1D quantizer (pinned in
test_oracle_quantize.py) on inputs where the 2D blocks reduce to 1D ones, and on
the transposed / transformed arrays; exact-rational nearest grid points; the
symmetry of 2D scaling under transposition; and the orthogonality that makes the
transform cancel in the weight-gradient product.
"""
from fractions import Fraction

import numpy as np
import scipy.linalg

import oracle

GRID = [0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0]


def unpack(codes: np.ndarray) -> np.ndarray:
    return np.stack([codes & 0xF, codes >> 4], axis=-1).reshape(codes.shape[0], -1)


def grid_value(code: int) -> float:
    v = GRID[code & 7]
    return -v if code & 8 else v


def bf16(x: np.ndarray) -> np.ndarray:
    """float32 -> bf16 bits, nearest-even."""
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def f32(bits: np.ndarray) -> np.ndarray:
    return (np.asarray(bits, dtype=np.uint32) << 16).view(np.float32)


def signs(seed: int) -> np.ndarray:
    return np.where(np.random.default_rng(seed).random(16) < 0.5, -1, 1).astype(np.int8)


# ----------------------------------------------------------------- R21: 2D scaling
def test_2d_equals_1d_when_every_row_holds_the_block_max():
    # each row of each 16 x 16 block carries the block's max magnitude, so every row's
    # 16-element amax is the 2D block's amax and the 2D store is the (pinned) 1D store
    rng = np.random.default_rng(1)
    R, C = 64, 96
    x = rng.standard_normal((R, C)).astype(np.float32)
    for bi in range(R // 16):
        for bj in range(C // 16):
            blk = x[16 * bi:16 * bi + 16, 16 * bj:16 * bj + 16]
            m = np.float32(np.abs(blk).max() * 1.5 + 0.1)
            for i in range(16):
                blk[i, (i * 7) % 16] = m if (i + bj) % 2 else -m
    codes, scales, _, _, a = oracle.quantize_2d(x)
    c1, s1, a1 = oracle.quantize(x)
    assert a == a1
    assert np.array_equal(codes, c1) and np.array_equal(scales, s1)


def test_2d_blocks_share_one_scale_and_codes_are_nearest_grid_points():
    rng = np.random.default_rng(2)
    R, C = 32, 64
    x = (rng.standard_normal((R, C)) * np.exp(rng.standard_normal((R, C)))).astype(np.float32)
    codes, scales, _, _, a32 = oracle.quantize_2d(x)
    q = unpack(codes)
    for bi in range(R // 16):
        for bj in range(C // 16):
            sb = scales[16 * bi:16 * bi + 16, bj]
            assert (sb == sb[0]).all()
            s = oracle.e4m3_value(int(sb[0]))
            denom = Fraction(float(np.float32(s) * np.float32(a32)))
            for r in range(16 * bi, 16 * bi + 16):
                for c in range(16 * bj, 16 * bj + 16):
                    y = Fraction(float(x[r, c])) / denom
                    got = Fraction(grid_value(int(q[r, c])))
                    if abs(y) >= 6:
                        assert abs(got) == 6
                        continue
                    best = min(abs(abs(y) - Fraction(g)) for g in GRID)
                    assert abs(abs(y) - abs(got)) <= best + abs(y) * Fraction(1, 2 ** 22), (r, c)
            # the block's largest element reaches the top of the grid (normal-range scale)
            if s >= 2.0 ** -6:
                blk = np.abs(x[16 * bi:16 * bi + 16, 16 * bj:16 * bj + 16])
                i, j = np.unravel_index(np.argmax(blk), blk.shape)
                assert abs(grid_value(int(q[16 * bi + i, 16 * bj + j]))) == 6


def test_2d_transposed_operand_is_the_2d_store_of_the_transpose():
    rng = np.random.default_rng(3)
    R, C = 48, 80
    x = bf16(rng.standard_normal((R, C)).astype(np.float32))
    codes, scales, codes_t, scales_t, a = oracle.quantize_2d(x)
    c2, s2, c2t, s2t, a2 = oracle.quantize_2d(np.ascontiguousarray(x.T))
    assert a == a2
    assert np.array_equal(codes_t, c2) and np.array_equal(scales_t, s2)
    assert np.array_equal(codes, c2t) and np.array_equal(scales, s2t)
    # and it is literally the transpose of the codes
    assert np.array_equal(unpack(codes_t), unpack(codes).T)


# ----------------------------------------------------------------- R22: the RHT
def test_rht_is_the_normalised_sylvester_hadamard_on_exact_inputs():
    H = scipy.linalg.hadamard(16)
    rng = np.random.default_rng(4)
    for seed in range(6):
        s = signs(seed)
        x = rng.integers(-100, 101, size=(8, 16)).astype(np.float32)
        got = oracle.rht16(x, s).reshape(8, 16)
        want = (x.astype(np.int64) * s) @ H.T / 4.0
        assert np.array_equal(got.astype(np.float64), want)


def test_rht_is_within_the_binary32_bound_and_orthogonal():
    H = scipy.linalg.hadamard(16).astype(np.float64)
    rng = np.random.default_rng(5)
    s = signs(5)
    x = (rng.standard_normal((200, 16)) * 3).astype(np.float32)
    got = oracle.rht16(x, s).reshape(200, 16).astype(np.float64)
    exact = (x.astype(np.float64) * s) @ H.T / 4.0
    bound = 4 * 2.0 ** -24 * np.abs(x.astype(np.float64)).sum(1, keepdims=True) / 4.0 * 1.01
    assert np.all(np.abs(got - exact) <= bound)
    # the inverse transform (H / 4, then the signs) returns the input
    back = (got @ H.T / 4.0) * s
    assert np.allclose(back, x, rtol=0, atol=1e-5)


# ----------------------------------------------------------------- transposed operand
def test_transposed_quantize_is_the_1d_quantize_of_the_transpose():
    rng = np.random.default_rng(6)
    R, C = 96, 40
    x = bf16(rng.standard_normal((R, C)).astype(np.float32))
    ct, st, a = oracle.quantize_t(x)
    c1, s1, a1 = oracle.quantize(np.ascontiguousarray(x.T))
    assert a == a1 and np.array_equal(ct, c1) and np.array_equal(st, s1)


def test_transposed_quantize_with_rht_is_the_1d_quantize_of_the_transformed_transpose():
    rng = np.random.default_rng(7)
    R, C = 64, 24
    x = bf16(rng.standard_normal((R, C)).astype(np.float32))
    s = signs(7)
    ct, st, a = oracle.quantize_t(x, sign=s)
    xt = np.ascontiguousarray(f32(x).T)
    yt = oracle.rht16(xt.reshape(-1), s).reshape(C, R)
    c1, s1, a1 = oracle.quantize(yt)
    assert a == a1 and np.array_equal(ct, c1) and np.array_equal(st, s1)


def test_rht_cancels_in_the_weight_gradient_product():
    # dW = dY^T X contracts over tokens; the same orthogonal transform on both operands
    # (blocks of 16 tokens, one sign vector) leaves the product unchanged up to the
    # transform's binary32 rounding.  A wrong sign, order or normalisation breaks this.
    rng = np.random.default_rng(8)
    M, N, K = 128, 32, 48
    dy = rng.standard_normal((M, N)).astype(np.float32)
    x = rng.standard_normal((M, K)).astype(np.float32)
    s = signs(8)
    a = oracle.rht16(np.ascontiguousarray(dy.T).reshape(-1), s).reshape(N, M).astype(np.float64)
    b = oracle.rht16(np.ascontiguousarray(x.T).reshape(-1), s).reshape(K, M).astype(np.float64)
    exact = dy.astype(np.float64).T @ x.astype(np.float64)
    assert np.abs(a @ b.T - exact).max() <= 1e-5 * np.abs(exact).max()
    # a different sign vector on one side does not cancel
    b2 = oracle.rht16(np.ascontiguousarray(x.T).reshape(-1), signs(9)).reshape(K, M).astype(np.float64)
    assert np.abs(a @ b2.T - exact).max() > 0.1 * np.abs(exact).max()


def test_quantized_weight_gradient_with_rht_is_within_the_format_error():
    # the NVFP4 weight gradient from transformed operands stays close to dY^T X
    rng = np.random.default_rng(10)
    M, N, K = 256, 32, 48
    dyb = bf16(rng.standard_normal((M, N)).astype(np.float32))
    xb = bf16(rng.standard_normal((M, K)).astype(np.float32))
    exact = f32(dyb).astype(np.float64).T @ f32(xb).astype(np.float64)
    s = signs(10)
    ca, sa, aa = oracle.quantize_t(dyb, sign=s)
    cb, sb, ab = oracle.quantize_t(xb, sign=s)
    A = oracle.dequant_f32(ca, sa, aa).astype(np.float64)
    B = oracle.dequant_f32(cb, sb, ab).astype(np.float64)
    # random signs in the sum cancel, so the relative error is that of single products (~0.1)
    assert np.abs(A @ B.T - exact).max() / np.abs(exact).max() < 0.25
