"""The 16384-token DiT linear stack, two layers chained on the GPU, each
hop's activation staying NVFP4 where the epilogue can produce it:
  QKV 3072->9216 (bf16; its V third, columns 6144.., quantized as the
  stand-in attention output) -> out-proj 3072->3072 with NVFP4 requant ->
  FFN up 3072->14336 with GELU and NVFP4 requant -> FFN down 14336->3072 with
  NVFP4 requant -> the next layer.
Every GEMM is checked on sampled rows against the oracle's fp64 GEMM on the
same NVFP4 operands (y within 2e-3 normwise, the bf16 output as bf16(y)), and
every requant bit for bit as the oracle's quantize of those rows of y with the
given output scale (calibrated by a first pass with out_amax)."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import GEMM_TOL, dev_bf16, f32_bits, host_bits, host_u8, normwise_err, require_gpu

pytestmark = pytest.mark.gpu

M = syn.STACK_M
ROWS = np.unique(np.concatenate([[0, 1, 255, 256, M - 1], np.random.default_rng(81).integers(0, M, 27)]))
ROWS_DEV = torch.from_numpy(ROWS).cuda() if torch.cuda.is_available() else None


def _weight(n, k, seed):
    bits = syn.normal_bf16((n, k), seed=seed, std=0.02)
    q = nv.quantize(dev_bf16(bits))
    oc, osc, oa = oracle.quantize(bits)
    torch.cuda.synchronize()
    assert np.array_equal(host_u8(q.codes), oc) and np.array_equal(host_u8(q.scales), oracle.swizzle(osc))
    return q, (oc, osc, oa)


def _rows_of(q: nv.NVFP4Tensor):
    """The sampled rows of a device NVFP4 tensor, as oracle operands."""
    codes = host_u8(q.codes.view(q.rows, -1)[ROWS_DEV])
    scales = oracle.unswizzle(host_u8(q.scales), q.rows, q.cols // 16)[ROWS]
    return codes, scales, np.float32(q.global_scale.item())


def _gemm_checked(qa, w, ow, *, act=0, requant=False):
    """Run one GEMM (with debug_y), check the sampled rows; return the device
    NVFP4 output (requant) or the bf16 output."""
    N = w.rows
    dy = torch.empty((qa.rows, N), dtype=torch.float32, device="cuda")
    out_q = None
    if requant:
        amax = torch.zeros(1, dtype=torch.float32, device="cuda")
        nv.gemm(qa, w, act=act, out_amax=amax)
        out_q = nv.empty_nvfp4(qa.rows, N)
        out_q.global_scale.copy_(amax / 2688.0)
        c = nv.gemm(qa, w, act=act, requant=out_q, debug_y=dy)
    else:
        c = nv.gemm(qa, w, act=act, debug_y=dy)
    torch.cuda.synchronize()
    y = dy[ROWS_DEV].cpu().numpy()
    ref, _ = oracle.gemm(_rows_of(qa), ow, act=act, want_bf16=False)
    assert normwise_err(y.astype(np.float64), ref) <= GEMM_TOL
    assert np.array_equal(host_bits(c[ROWS_DEV]), host_bits(dy[ROWS_DEV].to(torch.bfloat16)))
    if requant:
        a32 = np.float32(out_q.global_scale.item())
        codes, scales, _ = oracle.quantize(np.ascontiguousarray(y), a32)
        got = _rows_of(out_q)
        assert np.array_equal(got[0], codes) and np.array_equal(got[1], scales)
        return out_q
    return c


def test_two_layers_chained_sampled_rows():
    require_gpu()
    D, F = syn.STACK_LAYER[0].K, syn.STACK_LAYER[2].N
    x_bits = syn.activations_bf16(M, D, seed=80)
    a = nv.quantize(dev_bf16(x_bits))
    oc, osc, oa = oracle.quantize(x_bits)
    torch.cuda.synchronize()
    assert np.array_equal(host_u8(a.codes), oc) and f32_bits(a.global_scale.cpu().numpy()) == f32_bits(oa)
    for layer in range(2):
        s = 100 * (layer + 1)
        wqkv, oqkv = _weight(3 * D, D, s)
        wo, oo = _weight(D, D, s + 1)
        wup, oup = _weight(F, D, s + 2)
        wdn, odn = _weight(D, F, s + 3)
        qkv = _gemm_checked(a, wqkv, oqkv)
        v = qkv[:, 2 * D:].contiguous()
        av = nv.quantize(v)
        torch.cuda.synchronize()
        v_bits = host_bits(v)
        c2, s2, a2 = oracle.quantize(v_bits)
        assert f32_bits(av.global_scale.cpu().numpy()) == f32_bits(a2)
        assert np.array_equal(host_u8(av.codes), c2)
        assert np.array_equal(host_u8(av.scales), oracle.swizzle(s2))
        h1 = _gemm_checked(av, wo, oo, requant=True)
        h2 = _gemm_checked(h1, wup, oup, act=nv.ACT_GELU_TANH, requant=True)
        a = _gemm_checked(h2, wdn, odn, requant=True)
