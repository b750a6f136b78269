"""GPU parity of nvfp4_kv_append_rope: the keys' rotary embedding fused ahead of
their quantize (reading R24), codes, row-major scales and tensor scales bit for
bit against the oracle, V as the plain append; with K-smoothing the stored
channel means within the summation bound of the kernel's stated order around the
oracle's correctly rounded means, and the codes bit for bit against the oracle's
store built from those means; the dequant of the stored slot bit for bit too.  On the workload's 2640 x 24 x 128
chunk with its 3-frame x 22 x 40 angle table, and on ragged shapes."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import check_channel_means, dev_bf16, f32_bits, host_bits, host_u8, require_gpu

pytestmark = pytest.mark.gpu


def _dev_table(cs, sn):
    return (torch.from_numpy(np.ascontiguousarray(cs)).cuda(), torch.from_numpy(np.ascontiguousarray(sn)).cuda())


def _check(cache, slot, k, v, cs, sn, smooth_k=False, smooth_v=False, search=False):
    T, H, d = k.shape
    kmean = vmean = None
    if smooth_k:
        y = oracle.rope(k, cs, sn).reshape(T, -1)
        kmean = check_channel_means(cache.k_mean[slot], y, oracle.channel_mean_f32(y), "means of the turned keys")
    if smooth_v:
        vmean = check_channel_means(cache.v_mean[slot], syn.bf16_bits_to_f32(v).reshape(T, -1),
                                    oracle.channel_mean(v), "means of V")
    kc, ks, ka, km = oracle.kv_append_rope(k, cs, sn, smooth=smooth_k, search46=search, mean=kmean)
    if smooth_v:
        vc, vs, va, vm = oracle.kv_append_smooth(v, search46=search, mean=vmean)
    else:
        (vc, vs, va), vm = oracle.kv_append(v, search46=search), None
    for which, (c, s, a, m) in enumerate(((kc, ks, ka, km), (vc, vs, va, vm))):
        codes = cache.k_codes if which == 0 else cache.v_codes
        scales = cache.k_scales if which == 0 else cache.v_scales
        g = cache.k_global if which == 0 else cache.v_global
        assert f32_bits(g[slot].cpu().numpy()) == f32_bits(a), which
        assert np.array_equal(host_u8(codes[slot]), c.reshape(-1)), which
        assert np.array_equal(host_u8(scales[slot]), s.reshape(-1)), which
    kref = (oracle.kv_dequant_smooth(kc, ks, ka, km, T, H, d) if smooth_k else oracle.kv_dequant(kc, ks, ka, T, H, d))
    vref = (oracle.kv_dequant_smooth(vc, vs, va, vm, T, H, d) if smooth_v else oracle.kv_dequant(vc, vs, va, T, H, d))
    return kref, vref


@pytest.mark.parametrize("smooth_k,smooth_v,search", [(False, False, False), (True, False, True), (True, True, False)])
def test_full_chunk_with_the_3d_table(smooth_k, smooth_v, search):
    require_gpu()
    T, H, d = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    cs, sn = syn.rope_table_3d(*syn.KV_GRID, d, frame0=9)
    cache = nv.KVCache(2, T, H, d, scale_search=search, smooth_k=smooth_k, smooth_v=smooth_v)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=500)
    cache.append(1, dev_bf16(k), dev_bf16(v), rope=_dev_table(cs, sn))
    torch.cuda.synchronize()
    kref, vref = _check(cache, 1, k, v, cs, sn, smooth_k, smooth_v, search)
    ko, vo = cache.dequant(torch.tensor([1], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(ko)[0], kref) and np.array_equal(host_bits(vo)[0], vref)


def test_two_chunk_append_takes_the_register_kernel():
    """A 5280-token chunk (6 frames x 22 x 40; K + V = 32 M elements, past what the staged
    kernel holds in shared memory): the fused kernel with RoPE and both smoothings."""
    require_gpu()
    T, H, d = 2 * syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    f, hh, ww = syn.KV_GRID
    cs, sn = syn.rope_table_3d(2 * f, hh, ww, d, frame0=3)
    cache = nv.KVCache(1, T, H, d, smooth_k=True, smooth_v=True)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=501)
    cache.append(0, dev_bf16(k), dev_bf16(v), rope=_dev_table(cs, sn))
    torch.cuda.synchronize()
    _check(cache, 0, k, v, cs, sn, smooth_k=True, smooth_v=True)


@pytest.mark.parametrize("T,H,d", [(4, 3, 16), (12, 3, 16), (33, 2, 64), (64, 5, 32), (7, 1, 128)])
@pytest.mark.parametrize("smooth_k", [False, True])
def test_ragged_shapes_with_random_angles(T, H, d, smooth_k):
    """Fewer tokens than partial sums, channel counts that are not a multiple of 32
    (lanes past the channels in the means kernel), short last runs."""
    require_gpu()
    if (T * H * d) % 64:
        pytest.skip("T*H*d % 64")
    cs, sn = syn.rope_table(T, d, seed=T * 7 + d)
    cache = nv.KVCache(2, T, H, d, smooth_k=smooth_k)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=600 + T)
    cache.append(0, dev_bf16(k), dev_bf16(v), rope=_dev_table(cs, sn))
    torch.cuda.synchronize()
    kref, _ = _check(cache, 0, k, v, cs, sn, smooth_k)
    ko, _ = cache.dequant(torch.tensor([0], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(ko)[0], kref)


def test_identity_table_matches_the_plain_append():
    require_gpu()
    T, H, d = 96, 4, 64
    k, v = syn.kv_chunk_bf16(T, H, d, seed=700)
    plain = nv.KVCache(1, T, H, d)
    plain.append(0, dev_bf16(k), dev_bf16(v))
    roped = nv.KVCache(1, T, H, d)
    ones = torch.ones((T, d // 2), dtype=torch.float32, device="cuda")
    roped.append(0, dev_bf16(k), dev_bf16(v), rope=(ones, torch.zeros_like(ones)))
    torch.cuda.synchronize()
    for a, b in ((plain.k_codes, roped.k_codes), (plain.k_scales, roped.k_scales), (plain.k_global, roped.k_global),
                 (plain.v_codes, roped.v_codes)):
        assert torch.equal(a, b)


def test_bad_tables_are_rejected_on_the_host():
    require_gpu()
    T, H, d = 8, 2, 16
    cache = nv.KVCache(1, T, H, d)
    k, v = (dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, d, seed=1))
    with pytest.raises(ValueError):
        cache.append(0, k, v, rope=(torch.ones((T, d), device="cuda"), torch.zeros((T, d), device="cuda")))
    cc = ctypes.byref(cache.c())
    ws = cache.ws_append
    base = torch.zeros(T * d // 2 + 4, dtype=torch.float32, device="cuda")
    st = nv.lib().nvfp4_kv_append_rope(cc, 0, k.data_ptr(), v.data_ptr(), base.data_ptr() + 4, base.data_ptr(),
                                       ws.data_ptr(), ws.numel(), None)
    assert st == nv.ERR_MISALIGNED
    st = nv.lib().nvfp4_kv_append_rope(cc, 0, k.data_ptr(), v.data_ptr(), None, base.data_ptr(),
                                       ws.data_ptr(), ws.numel(), None)
    assert st == nv.ERR_INVALID_ARG
