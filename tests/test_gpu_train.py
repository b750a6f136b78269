"""GPU parity of the training-side NVFP4 operands against the oracle (bit for
bit): nvfp4_quantize_2d (16 x 16 block scaling of weights, both the row-wise
and the transposed operand) and nvfp4_quantize_t (the transposed operand of
the weight-gradient GEMM, with and without the 16-point Random Hadamard
Transform), then the weight-gradient and data-gradient GEMMs on those
operands through nvfp4_gemm (reading R12's 2e-3 normwise bound against the
oracle's fp64 GEMM of the same operands)."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import GEMM_TOL, dev_bf16, f32_bits, host_u8, normwise_err, require_gpu

pytestmark = pytest.mark.gpu

SIGN = np.array([1, -1, -1, 1, 1, 1, -1, 1, -1, -1, 1, -1, 1, 1, -1, -1], np.int8)


def _check(q, codes, scales, alpha):
    assert f32_bits(q.global_scale.cpu().numpy()) == f32_bits(alpha)
    assert np.array_equal(host_u8(q.codes), codes)
    assert np.array_equal(host_u8(q.scales), oracle.swizzle(scales))


def _q2d(bits, alpha=None):
    gs = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    a, t = nv.quantize_2d(dev_bf16(bits), global_scale=gs)
    oc, osc, oct_, ost, oa = oracle.quantize_2d(bits, alpha)
    torch.cuda.synchronize()
    _check(a, oc, osc, oa)
    _check(t, oct_, ost, oa)
    return a, t, (oc, osc, oa), (oct_, ost, oa)


def _qt(bits, sign=None, alpha=None):
    gs = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    q = nv.quantize_t(dev_bf16(bits), rht_sign=sign, global_scale=gs)
    oc, osc, oa = oracle.quantize_t(bits, sign=sign, alpha=alpha)
    torch.cuda.synchronize()
    _check(q, oc, osc, oa)
    return q, (oc, osc, oa)


def test_2d_weight_at_the_qkv_size():
    """The QKV weight 9216 x 3072: both operands and the tensor scale bit for bit."""
    require_gpu()
    _q2d(syn.normal_bf16((9216, 3072), seed=3, std=0.02))


@pytest.mark.parametrize("rows,cols", [(64, 64), (192, 320), (320, 192)])
def test_2d_ragged_shapes_and_padding(rows, cols):
    require_gpu()
    _q2d(syn.activations_bf16(rows, cols, seed=rows + cols))


def test_2d_given_scale_that_saturates_and_flushes():
    require_gpu()
    bits = syn.activations_bf16(128, 128, seed=5)
    _q2d(bits, alpha=1e-4)   # most blocks saturate at 448
    _q2d(bits, alpha=1e3)    # most blocks flush to zero
    _q2d(np.zeros((64, 64), np.uint16))


@pytest.mark.parametrize("sign", [None, SIGN])
def test_transposed_operand_at_the_qkv_size(sign):
    """Activations 4096 x 3072 (tokens x features) as the weight-gradient operand."""
    require_gpu()
    _qt(syn.activations_bf16(4096, 3072, seed=6), sign)


@pytest.mark.parametrize("rows,cols", [(64, 16), (192, 48), (128, 200 - 200 % 16), (256, 1040)])
@pytest.mark.parametrize("sign", [None, SIGN])
def test_transposed_operand_ragged(rows, cols, sign):
    require_gpu()
    _qt(syn.activations_bf16(rows, cols, seed=rows * 7 + cols), sign)


def test_transposed_operand_given_scale_and_zero():
    require_gpu()
    bits = syn.activations_bf16(128, 64, seed=8)
    _qt(bits, SIGN, alpha=2e-4)
    _qt(np.zeros((64, 32), np.uint16), SIGN)


def _gemm_checked(qa, qb, oa, ob):
    M, N = qa.rows, qb.rows
    dy = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.gemm(qa, qb, debug_y=dy)
    torch.cuda.synchronize()
    ref, _ = oracle.gemm(oa, ob, want_bf16=False)
    err = normwise_err(dy.cpu().numpy().astype(np.float64), ref)
    assert err <= GEMM_TOL, err
    return ref


def test_weight_gradient_gemm_on_rht_operands():
    """dW [N x K] = dY^T X over 1024 tokens: both operands through the RHT with the
    same signs, the GEMM against the oracle on the same operands, and the result
    close to the unquantized dY^T X (the transform cancels)."""
    require_gpu()
    M, N, K = 1024, 256, 384
    dyb = syn.activations_bf16(M, N, seed=9)
    xb = syn.activations_bf16(M, K, seed=10)
    qa, oa = _qt(dyb, SIGN)
    qb, ob = _qt(xb, SIGN)
    ref = _gemm_checked(qa, qb, oa, ob)
    exact = syn.bf16_bits_to_f32(dyb).astype(np.float64).T @ syn.bf16_bits_to_f32(xb).astype(np.float64)
    assert normwise_err(ref, exact) < 0.25


def test_data_gradient_gemm_on_the_2d_transposed_weight():
    """dX [M x K] = dY W with W [N x K] 2D-scaled once: the GEMM reads W^T's operand."""
    require_gpu()
    M, N, K = 512, 384, 256
    dyb = syn.activations_bf16(M, N, seed=11)
    wb = syn.normal_bf16((N, K), seed=12, std=0.02)
    _, wt, _, owt = _q2d(wb)
    qa = nv.quantize(dev_bf16(dyb))
    oa = oracle.quantize(dyb)
    torch.cuda.synchronize()
    _check(qa, *oa)
    _gemm_checked(qa, wt, oa, owt)
