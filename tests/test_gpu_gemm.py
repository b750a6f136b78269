"""GPU parity of nvfp4_gemm against the oracle's fp64 GEMM.

Metric (reading R12): max_ij |y - ref| / max_ij |ref| <= 2e-3, where y is the
kernel's binary32 result (accumulation and epilogue, before the output store;
written to the debug output) and ref the oracle's fp64 result on the same
NVFP4 operands (the operands are checked bit-exact here too).  The bf16
output is then checked bit for bit as the nearest-even bf16 of y, and the
fused requant bit for bit as the oracle's quantize of y (reading R13).  The
bf16 store alone can move a value by 2^-8 relative, so the 2e-3 bound is not
applied to it.
"""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import GEMM_TOL, bf16_to_f64, dev_bf16, f32_bits, host_bits, host_u8, normwise_err, require_gpu

pytestmark = pytest.mark.gpu


def _qboth(bits, alpha=None):
    """Quantize on the GPU and with the oracle; assert they agree; return both."""
    xd = dev_bf16(bits)
    gs = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    q = nv.quantize(xd, global_scale=gs)
    oc, osc, oa = oracle.quantize(bits, alpha)
    torch.cuda.synchronize()
    assert np.array_equal(host_u8(q.codes), oc)
    assert np.array_equal(host_u8(q.scales), oracle.swizzle(osc))
    assert f32_bits(q.global_scale.cpu().numpy()) == f32_bits(oa)
    return q, (oc, osc, oa)


def _gemm_case(M, N, K, seed, **ep):
    a = syn.activations_bf16(M, K, seed=seed)
    b = syn.normal_bf16((N, K), seed=seed + 1, std=0.02)
    qa, oa = _qboth(a)
    qb, ob = _qboth(b)
    return qa, oa, qb, ob


def _run_checked(qa, qb, oa, ob, rows=None, out=None, **ep):
    """Run nvfp4_gemm with the debug output, check y against the oracle at
    GEMM_TOL and the bf16 output against bf16(y) exactly; return (c, y)."""
    M, N = qa.rows, qb.rows
    dy = torch.empty((M, N), dtype=torch.float32, device="cuda")
    dk = {k: (dev_bf16(v) if isinstance(v, np.ndarray) else v) for k, v in ep.items()}
    c = nv.gemm(qa, qb, out=out, debug_y=dy, **dk)
    torch.cuda.synchronize()
    ref, _ = oracle.gemm(oa, ob, rows=rows, want_bf16=False, **ep)
    y = dy.cpu().numpy()
    ys = y if rows is None else y[rows]
    err = normwise_err(ys.astype(np.float64), ref)
    assert np.isfinite(ys).all()
    assert err <= GEMM_TOL, err
    cb = host_bits(c if out is None else out)
    want = host_bits(dy.to(torch.bfloat16))
    assert np.array_equal(cb, want), "bf16 output is not the nearest-even bf16 of y"
    return c, y, err


@pytest.mark.parametrize("M,N,K", [(64, 128, 256)])
def test_tiny_workload(M, N, K):
    require_gpu()
    a = syn.tiny_a_bf16(M, K, seed=0)
    b = syn.normal_bf16((N, K), seed=1)
    qa, oa = _qboth(a)
    qb, ob = _qboth(b)
    c, y, _ = _run_checked(qa, qb, oa, ob)
    exact = bf16_to_f64(oracle.gemm_exact_bf16(oa, ob))
    assert normwise_err(y.astype(np.float64), exact) <= GEMM_TOL


def _lossless(rows, cols, seed):
    g = np.random.default_rng(seed)
    grid = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6], np.float64)
    v = grid[g.integers(0, 8, size=(rows, cols))] * g.choice([-1.0, 1.0], size=(rows, cols))
    v[:, ::16] = 6.0 * g.choice([-1.0, 1.0], size=(rows, cols // 16))
    e = g.integers(-3, 1, size=(rows, cols // 16)).astype(np.float64)
    return v * np.repeat(2.0 ** e, 16, axis=1)


@pytest.mark.parametrize("M,N,K", [(128, 256, 256), (200, 136, 320), (64, 512, 1024)])
def test_lossless_operands_give_textbook_matmul(M, N, K):
    # Exact operands: any error in code nibble order, scale-tile layout,
    # operand transposition or K stepping shows up as an O(1) error.
    require_gpu()
    a = _lossless(M, K, 1000 + M)
    b = _lossless(N, K, 2000 + N)
    alpha = np.float32(2.0 ** -8)
    qa, _ = _qboth(syn.f32_to_bf16_bits(a.astype(np.float32)), alpha)
    qb, _ = _qboth(syn.f32_to_bf16_bits(b.astype(np.float32)), alpha)
    y = torch.empty((M, N), dtype=torch.float32, device="cuda")
    nv.gemm(qa, qb, debug_y=y)
    # s * a32 = 2^e exactly, so a32_A a32_B (A_q S_A)(B_q S_B)^T = A B^T
    ref = a @ b.T
    got = y.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(got - ref)) <= 1e-6 * np.max(np.abs(ref))


def test_qkv_full_size_sampled_rows():
    require_gpu()
    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=2)
    bias = syn.normal_bf16((N,), seed=4, std=0.02)
    rows = np.unique(np.concatenate([[0, 1, 127, 128, M - 1],
                                     np.random.default_rng(5).integers(0, M, 59)]))
    _run_checked(qa, qb, oa, ob, rows=rows, bias=bias)


@pytest.mark.parametrize("M,N,K", [(1, 8, 64), (100, 136, 320), (130, 264, 512), (300, 520, 192),
                                   (257, 256, 1024), (129, 1000, 64)])
def test_ragged_shapes(M, N, K):
    require_gpu()
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=M + N + K)
    ldc = (N + 7) // 8 * 8 + 8
    buf = torch.full((M, ldc), float("nan"), dtype=torch.bfloat16, device="cuda")
    _run_checked(qa, qb, oa, ob, out=buf[:, :N])
    assert torch.isnan(buf[:, N:]).all()  # nothing written past N


@pytest.mark.parametrize("M,N,K", [(100, 264, 4160), (300, 520, 4352), (256, 256, 8192)])
def test_long_k_shapes(M, N, K):
    """More than 16 K-stages per tile: the kernel variant with three scale-copy
    warps (single-CTA and CTA-pair tiles, a one-k-block K tail)."""
    require_gpu()
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=M + N + K)
    bias = syn.normal_bf16((N,), seed=7, std=0.02)
    _run_checked(qa, qb, oa, ob, bias=bias)


def _sampled_rows(M, seed):
    return np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, M - 1],
                                     np.random.default_rng(seed).integers(0, M, 41)]))


def test_ffn_full_size_up_gelu_requant_then_down_sampled_rows():
    """DiT FFN pair at full size (8192 tokens, 3072 -> 14336 -> 3072): the
    up-projection with GELU and the NVFP4 requant epilogue, then the
    down-projection reading that NVFP4 output; checked on sampled rows."""
    require_gpu()
    M, D, F = syn.FFN_UP.M, syn.FFN_UP.K, syn.FFN_UP.N
    qa, oa = _qboth(syn.activations_bf16(M, D, seed=51))
    qu, ou = _qboth(syn.normal_bf16((F, D), seed=52, std=0.02))
    qd, od = _qboth(syn.normal_bf16((D, F), seed=53, std=0.02))
    rows = _sampled_rows(M, 54)
    # output scale of the up-projection: delayed scaling from a calibration pass
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, out_amax=amax)
    h = nv.empty_nvfp4(M, F)
    h.global_scale.copy_(amax / 2688.0)
    dy = torch.empty((M, F), dtype=torch.float32, device="cuda")
    c = nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, requant=h, debug_y=dy)
    torch.cuda.synchronize()
    ref, _ = oracle.gemm(oa, ou, act=1, rows=rows, want_bf16=False)
    y = dy.cpu().numpy()
    assert normwise_err(y[rows].astype(np.float64), ref) <= GEMM_TOL
    assert np.array_equal(host_bits(c)[rows], host_bits(dy.to(torch.bfloat16))[rows])
    # requant of the sampled rows: the oracle's quantize of y with the given scale (row-local)
    ha32 = np.float32(h.global_scale.item())
    codes, scales, _ = oracle.quantize(np.ascontiguousarray(y[rows]), ha32)
    assert np.array_equal(host_u8(h.codes)[rows], codes)
    sc_dev = oracle.unswizzle(host_u8(h.scales), M, F // 16)
    assert np.array_equal(sc_dev[rows], scales)
    # down-projection over the NVFP4 hidden state (K = 14336: the long-K variant)
    oh = (host_u8(h.codes), sc_dev, ha32)
    _run_checked(h, qd, oh, od, rows=rows)


def test_stack_layer_qkv_16384_tokens_sampled_rows():
    """The QKV projection of the 16384-token linear stack (3072 -> 9216)."""
    require_gpu()
    M, N, K = 16384, 9216, 3072
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=61)
    bias = syn.normal_bf16((N,), seed=62, std=0.02)
    _run_checked(qa, qb, oa, ob, rows=_sampled_rows(M, 63), bias=bias)


def test_epilogue_bias_gelu_modulate_gate_residual():
    require_gpu()
    M, N, K = 256, 512, 512
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=11)
    bias = syn.normal_bf16((N,), seed=12, std=0.1)
    ms = syn.normal_bf16((N,), seed=13, std=0.1)
    sh = syn.normal_bf16((N,), seed=14, std=0.1)
    gt = syn.normal_bf16((N,), seed=15, std=0.5)
    res = syn.normal_bf16((M, N), seed=16)
    for kw in (dict(bias=bias, act=nv.ACT_GELU_TANH), dict(mod_scale=ms, mod_shift=sh),
               dict(bias=bias, gate=gt, residual=res), dict(bias=bias, act=1, mod_scale=ms, mod_shift=sh,
                                                             gate=gt, residual=res)):
        _run_checked(qa, qb, oa, ob, **kw)


@pytest.mark.parametrize("M,N,K", [(256, 512, 256), (200, 320, 512)])
def test_requant_epilogue_bit_exact_given_prequant_values(M, N, K):
    require_gpu()
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=21)
    bias = syn.normal_bf16((N,), seed=22, std=0.1)
    y_ref, _ = oracle.gemm(oa, ob, bias=bias, act=1, want_bf16=False)
    out_a32 = np.float32(np.max(np.abs(y_ref)) / 2688.0)
    rq = nv.empty_nvfp4(M, N)
    rq.global_scale.fill_(float(out_a32))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    dy = torch.empty((M, N), dtype=torch.float32, device="cuda")
    c = nv.gemm(qa, qb, bias=dev_bf16(bias), act=nv.ACT_GELU_TANH, requant=rq, out_amax=amax, debug_y=dy)
    torch.cuda.synchronize()
    y = dy.cpu().numpy()
    assert normwise_err(y.astype(np.float64), y_ref) <= GEMM_TOL
    assert np.array_equal(host_bits(c), host_bits(dy.to(torch.bfloat16)))
    codes, scales, _ = oracle.quantize(np.ascontiguousarray(y), out_a32)
    assert np.array_equal(host_u8(rq.codes), codes)
    assert np.array_equal(host_u8(rq.scales), oracle.swizzle(scales))
    assert float(amax.item()) == float(np.max(np.abs(y)))
    # requant alone (no bf16 output) gives the same codes
    rq2 = nv.empty_nvfp4(M, N)
    rq2.global_scale.fill_(float(out_a32))
    nv.gemm(qa, qb, bias=dev_bf16(bias), act=nv.ACT_GELU_TANH, requant=rq2, bf16_out=False)
    torch.cuda.synchronize()
    assert torch.equal(rq2.codes, rq.codes) and torch.equal(rq2.scales, rq.scales)


def test_ffn_pair_up_requant_feeds_down():
    require_gpu()
    M, D, F = 512, 768, 1536
    a = syn.activations_bf16(M, D, seed=31)
    wu = syn.normal_bf16((F, D), seed=32, std=0.02)
    wd = syn.normal_bf16((D, F), seed=33, std=0.02)
    qa, oa = _qboth(a)
    qu, ou = _qboth(wu)
    qd, od = _qboth(wd)
    # calibration pass: out_amax of the up-projection gives its output scale
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, out_amax=amax)
    h = nv.empty_nvfp4(M, F)
    h.global_scale.copy_(amax / 2688.0)
    nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, requant=h, bf16_out=False)
    torch.cuda.synchronize()
    oh = (host_u8(h.codes), oracle.unswizzle(host_u8(h.scales), M, F // 16), np.float32(h.global_scale.item()))
    _run_checked(h, qd, oh, od)
    # and the whole chain stays close to the fp64 chain of the oracle
    yu, _ = oracle.gemm(oa, ou, act=1, want_bf16=False)
    assert abs(float(amax.item()) - np.max(np.abs(yu))) <= 2e-3 * np.max(np.abs(yu))


def test_bounded_wait_records_timeout_and_context_survives():
    require_gpu()
    qa, oa, qb, ob = _gemm_case(128, 256, 256, seed=41)
    ws = nv.workspace(nv.OP_GEMM)
    nv.gemm(qa, qb, debug_flags=nv.DBG_SKIP_LOADS, wait_limit_us=50000, ws=ws)
    code, info = nv.read_device_error(ws)
    assert code == nv.ERR_TIMEOUT and info in (2, 3, 4)
    _run_checked(qa, qb, oa, ob)
    nv.gemm(qa, qb, ws=ws)
    code, _ = nv.read_device_error(ws)
    assert code == nv.OK


@pytest.mark.parametrize("M,N,K,col0,cols", [(200, 512, 256, 128, 192), (300, 9216 // 8, 512, 768, 384),
                                            (129, 256, 256, 0, 64)])
def test_requant_of_a_column_window(M, N, K, col0, cols):
    """The requant (and out_amax) of columns col0 .. col0 + cols - 1 only, as an
    [M, cols] operand (a QKV projection's V third): bit for bit the oracle's
    quantize of those columns of y; the bf16 output still covers every column."""
    require_gpu()
    qa, oa, qb, ob = _gemm_case(M, N, K, seed=91 + col0)
    bias = syn.normal_bf16((N,), seed=92, std=0.1)
    y_ref, _ = oracle.gemm(oa, ob, bias=bias, want_bf16=False)
    out_a32 = np.float32(np.max(np.abs(y_ref[:, col0:col0 + cols])) / 2688.0)
    rq = nv.empty_nvfp4(M, cols)
    rq.global_scale.fill_(float(out_a32))
    amax = torch.zeros(1, dtype=torch.float32, device="cuda")
    dy = torch.empty((M, N), dtype=torch.float32, device="cuda")
    c = nv.gemm(qa, qb, bias=dev_bf16(bias), requant=rq, out_amax=amax, debug_y=dy, out_window=(col0, cols))
    torch.cuda.synchronize()
    y = dy.cpu().numpy()
    assert normwise_err(y.astype(np.float64), y_ref) <= GEMM_TOL
    assert np.array_equal(host_bits(c), host_bits(dy.to(torch.bfloat16)))
    yw = np.ascontiguousarray(y[:, col0:col0 + cols])
    codes, scales, _ = oracle.quantize(yw, out_a32)
    assert np.array_equal(host_u8(rq.codes), codes)
    assert np.array_equal(host_u8(rq.scales), oracle.swizzle(scales))
    assert float(amax.item()) == float(np.max(np.abs(yw)))
    # the same window without a bf16 output gives the same operand
    rq2 = nv.empty_nvfp4(M, cols)
    rq2.global_scale.fill_(float(out_a32))
    nv.gemm(qa, qb, bias=dev_bf16(bias), requant=rq2, bf16_out=False, out_window=(col0, cols))
    torch.cuda.synchronize()
    assert torch.equal(rq2.codes, rq.codes) and torch.equal(rq2.scales, rq.scales)
