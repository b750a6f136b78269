"""Pins of the oracle's fp64 GEMM, epilogue and KV-cache store.

- the fp64 GEMM equals an exact rational GEMM (integer arithmetic, one final
  rounding) on tiny inputs, the workload's 64x128x256 case included;
- lossless special case: operands built on the E2M1 grid with power-of-two
  block scales quantize without error, so the NVFP4 GEMM must equal numpy's
  float64 matmul A @ B^T of the original values (catches a transposed operand,
  a lost sign, a dropped tensor or block scale);
- the GELU epilogue equals torch's tanh-form GELU; modulate / gate / residual
  reduce to the identity for scale 0, shift 0, gate 1, residual 0 and add
  exactly otherwise;
- KV bytes per chunk equal the 9/8 * T_c * H * d of "LongLive-2.0：用 NVFP4
  并行底座做长视频生成" (yingwang.github.io reading note), section 二 方法 /
  "推理底座"; the bf16 dequant equals torch's bf16 rounding of the binary32
  dequant (R10).
"""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import synthetic as syn


def _q(x, alpha=None):
    return oracle.quantize(x, alpha)


@pytest.mark.parametrize("M,N,K,seed", [(64, 128, 256, 0), (1, 1, 16, 1), (7, 5, 48, 2),
                                        (33, 17, 64, 3), (64, 64, 160, 4)])
def test_fp64_gemm_equals_exact_rational(M, N, K, seed):
    if (M, N, K) == (64, 128, 256):
        a = syn.tiny_a_bf16(M, K, seed=0)
        b = syn.normal_bf16((N, K), seed=1)
    else:
        a = syn.activations_bf16(M, K, seed=seed)
        b = syn.normal_bf16((N, K), seed=seed + 100, std=0.02)
    qa, qb = _q(a), _q(b)
    _, fp = oracle.gemm(qa, qb)
    ex = oracle.gemm_exact_bf16(qa, qb)
    assert (fp == ex).all()


def _lossless_operand(rows, cols, seed):
    """Values v * 2^e with v on the E2M1 grid and one power-of-two e per
    16-block, each block holding a +-6 so its scale is exactly 2^(e+8) when the
    tensor scale is 2^-8."""
    g = np.random.default_rng(seed)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    v = grid[g.integers(0, 8, size=(rows, cols))] * g.choice([-1.0, 1.0], size=(rows, cols))
    v[:, ::16] = 6.0 * g.choice([-1.0, 1.0], size=(rows, cols // 16))
    e = g.integers(-10, 1, size=(rows, cols // 16)).astype(np.float64)
    x = v * np.repeat(2.0 ** e, 16, axis=1)
    return x


@pytest.mark.parametrize("M,N,K", [(64, 128, 256), (19, 37, 96), (128, 8, 512)])
def test_lossless_inputs_give_textbook_matmul(M, N, K):
    a = _lossless_operand(M, K, 10 + M)
    b = _lossless_operand(N, K, 20 + N)
    alpha = np.float32(2.0 ** -8)
    qa = _q(syn.f32_to_bf16_bits(a.astype(np.float32)), alpha)
    qb = _q(syn.f32_to_bf16_bits(b.astype(np.float32)), alpha)
    # the quantization itself is lossless
    assert (oracle.dequant_f32(*qa) == a).all() and (oracle.dequant_f32(*qb) == b).all()
    y, _ = oracle.gemm(qa, qb, want_bf16=False)
    assert np.array_equal(y, a @ b.T)


def test_epilogue_gelu_matches_torch():
    a = syn.activations_bf16(16, 128, seed=5)
    b = syn.normal_bf16((24, 128), seed=6, std=0.1)
    qa, qb = _q(a), _q(b)
    bias = syn.normal_bf16((24,), seed=7, std=0.5)
    y0, _ = oracle.gemm(qa, qb, bias=bias)
    y1, _ = oracle.gemm(qa, qb, bias=bias, act=1)
    ref = torch.nn.functional.gelu(torch.from_numpy(y0), approximate="tanh").numpy()
    np.testing.assert_allclose(y1, ref, rtol=1e-13, atol=1e-15)
    yp, _ = oracle.gemm(qa, qb)
    np.testing.assert_array_equal(y0, yp + syn.bf16_bits_to_f32(bias).astype(np.float64)[None, :])


def test_epilogue_modulate_gate_residual_special_cases():
    a = syn.activations_bf16(8, 64, seed=8)
    b = syn.normal_bf16((16, 64), seed=9, std=0.1)
    qa, qb = _q(a), _q(b)
    z = np.zeros(16, np.uint16)
    one = syn.f32_to_bf16_bits(np.ones(16, np.float32))
    two = syn.f32_to_bf16_bits(np.full(16, 2.0, np.float32))
    res0 = np.zeros((8, 16), np.uint16)
    y, _ = oracle.gemm(qa, qb)
    y_id, _ = oracle.gemm(qa, qb, mod_scale=z, mod_shift=z, gate=one, residual=res0)
    np.testing.assert_array_equal(y, y_id)
    y_mod, _ = oracle.gemm(qa, qb, mod_scale=one, mod_shift=two)     # y * 2 + 2
    np.testing.assert_array_equal(y_mod, 2.0 * y + 2.0)
    res = syn.normal_bf16((8, 16), seed=10)
    y_gr, _ = oracle.gemm(qa, qb, gate=two, residual=res)             # res + 2 y
    np.testing.assert_array_equal(y_gr, syn.bf16_bits_to_f32(res).astype(np.float64) + 2.0 * y)


def test_sampled_rows_equal_full_rows():
    a = syn.activations_bf16(40, 64, seed=12)
    b = syn.normal_bf16((24, 64), seed=13, std=0.02)
    qa, qb = _q(a), _q(b)
    yf, of = oracle.gemm(qa, qb)
    rows = [39, 0, 17, 17]
    ys, os_ = oracle.gemm(qa, qb, rows=rows)
    np.testing.assert_array_equal(ys, yf[rows])
    np.testing.assert_array_equal(os_, of[rows])


def test_kv_bytes_match_page(golden):
    for T, H, d, bf16_bytes, nv_bytes in golden("kv_bytes.txt"):
        T, H, d = int(T), int(H), int(d)
        assert 2 * 2 * T * H * d == int(bf16_bytes)
        assert 2 * oracle.kv_slot_bytes(T, H, d) == int(nv_bytes)


def test_kv_append_dequant_roundtrip():
    k, v = syn.kv_chunk_bf16(16, 4, 128, seed=3)
    for x in (k, v):
        codes, scales, a32 = oracle.kv_append(x)
        assert codes.shape == (64, 64) and scales.shape == (64, 8)
        assert codes.nbytes + scales.nbytes == oracle.kv_slot_bytes(16, 4, 128)
        c2, s2, a2 = oracle.quantize(x.reshape(64, 128))
        assert a2 == a32 and (c2 == codes).all() and (s2 == scales).all()
        f32 = oracle.dequant_f32(codes, scales, a32)
        bf = oracle.kv_dequant(codes, scales, a32, 16, 4, 128).reshape(64, 128)
        ref = torch.from_numpy(f32).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
        assert (bf == ref).all()
        # error bound of the format: within one E2M1 half-gap of the block scale
        xf = syn.bf16_bits_to_f32(x.reshape(64, 128))
        s = np.vectorize(oracle.e4m3_value)(scales).repeat(16, axis=1) * np.float64(a32)
        assert (np.abs(xf - f32) <= 1.0 * s * (1 + 1e-6) + 1e-30).all()
