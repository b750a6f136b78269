"""GPU parity of the NVFP4 KV-cache store: nvfp4_kv_append (codes, row-major
scales and per-slot tensor scales bit for bit) and nvfp4_kv_dequant (bf16 bit
for bit), on the workload's 2640 x 24 x 128 chunk and on small rings."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import check_channel_means, dev_bf16, f32_bits, host_bits, host_u8, require_gpu

pytestmark = pytest.mark.gpu


def _oracle_slot(x):
    T, H, d = x.shape
    return oracle.kv_append(x)


def _check_slot(cache, slot, x, which):
    codes, scales, a32 = _oracle_slot(x)
    c = cache.k_codes if which == 0 else cache.v_codes
    s = cache.k_scales if which == 0 else cache.v_scales
    g = cache.k_global if which == 0 else cache.v_global
    assert f32_bits(g[slot].cpu().numpy()) == f32_bits(a32)
    assert np.array_equal(host_u8(c[slot]), codes.reshape(-1))
    assert np.array_equal(host_u8(s[slot]), scales.reshape(-1))
    return codes, scales, a32


def test_full_chunk_append_and_dequant():
    require_gpu()
    T, H, d = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    cache = nv.KVCache(3, T, H, d)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=0)
    cache.append(2, dev_bf16(k), dev_bf16(v))
    torch.cuda.synchronize()
    for which, x in ((0, k), (1, v)):
        codes, scales, a32 = _check_slot(cache, 2, x, which)
        ref = oracle.kv_dequant(codes, scales, a32, T, H, d)
        slots = torch.tensor([2], dtype=torch.int32, device="cuda")
        ko, vo = cache.dequant(slots)
        got = host_bits(ko if which == 0 else vo)[0]
        assert np.array_equal(got, ref)
    assert cache.k_codes[2].numel() + cache.k_scales[2].numel() == oracle.kv_slot_bytes(T, H, d)


@pytest.mark.parametrize("T,H,d", [(16, 4, 128), (3, 2, 64), (8, 24, 16)])
def test_ring_of_slots_and_page_table(T, H, d):
    require_gpu()
    n_slots = 5
    cache = nv.KVCache(n_slots, T, H, d)
    latest = {}
    for step in range(8):
        k, v = syn.kv_chunk_bf16(T, H, d, seed=100 + step)
        slot = step % n_slots
        cache.append(slot, dev_bf16(k), dev_bf16(v))
        latest[slot] = (k, v)
    torch.cuda.synchronize()
    order = [3, 4, 0, 1, 2, 3]
    slots = torch.tensor(order, dtype=torch.int32, device="cuda")
    ko, vo = cache.dequant(slots)
    ko, vo = host_bits(ko), host_bits(vo)
    for i, s in enumerate(order):
        for which, x in enumerate(latest[s]):
            codes, scales, a32 = _check_slot(cache, s, x, which)
            ref = oracle.kv_dequant(codes, scales, a32, T, H, d)
            assert np.array_equal((ko if which == 0 else vo)[i], ref), (i, s, which)


def test_out_of_range_slot_is_reported():
    require_gpu()
    T, H, d = 4, 2, 64
    cache = nv.KVCache(2, T, H, d)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=9)
    cache.append(0, dev_bf16(k), dev_bf16(v))
    slots = torch.tensor([0, 7, 0], dtype=torch.int32, device="cuda")
    ko = torch.zeros((3, T, H, d), dtype=torch.bfloat16, device="cuda")
    vo = torch.zeros((3, T, H, d), dtype=torch.bfloat16, device="cuda")
    cache.dequant(slots, ko, vo)
    code, info = nv.read_device_error(cache.ws_dequant)
    assert code == nv.ERR_DEVICE and info == 1
    assert not bool(ko[1].view(torch.int16).any())   # that chunk is left unwritten
    assert bool((ko[0] == ko[2]).all())
    code, _ = nv.read_device_error(cache.ws_dequant)  # the record was cleared
    assert code == nv.OK


def test_full_chunk_append_with_scale_search():
    """KV append with the adaptive scale search ({4, 6}) on the full chunk: codes,
    scales and tensor scales bit for bit against the oracle, and the bf16 dequant."""
    require_gpu()
    T, H, d = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    cache = nv.KVCache(2, T, H, d, scale_search=True)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=4)
    cache.append(1, dev_bf16(k), dev_bf16(v))
    torch.cuda.synchronize()
    for which, x in ((0, k), (1, v)):
        codes, scales, a32 = oracle.kv_append(x, search46=True)
        c = cache.k_codes if which == 0 else cache.v_codes
        s = cache.k_scales if which == 0 else cache.v_scales
        g = cache.k_global if which == 0 else cache.v_global
        assert f32_bits(g[1].cpu().numpy()) == f32_bits(a32)
        assert np.array_equal(host_u8(c[1]), codes.reshape(-1))
        assert np.array_equal(host_u8(s[1]), scales.reshape(-1))
    slots = torch.tensor([1], dtype=torch.int32, device="cuda")
    ko, vo = cache.dequant(slots)
    torch.cuda.synchronize()
    for x, o in ((k, ko), (v, vo)):
        codes, scales, a32 = oracle.kv_append(x, search46=True)
        want = oracle.kv_dequant(codes, scales, a32, T, H, d)
        assert np.array_equal(host_bits(o[0]), want)


def _check_smoothed(cache, slot, x, which, smoothed, search):
    """One slot's K or V against the oracle: the stored channel means (when
    smoothed) within the summation bound of the kernel's stated order around the
    oracle's correctly rounded means, then codes, scales and tensor scale bit for
    bit against the oracle's smoothed store built from the kernel's means; returns
    what the oracle's dequant needs."""
    T, H, d = x.shape
    if smoothed:
        m = cache.k_mean if which == 0 else cache.v_mean
        km = check_channel_means(m[slot], syn.bf16_bits_to_f32(x).reshape(T, -1), oracle.channel_mean(x))
        codes, scales, a32, mean = oracle.kv_append_smooth(x, search46=search, mean=km)
    else:
        codes, scales, a32 = oracle.kv_append(x, search46=search)
        mean = None
    c = cache.k_codes if which == 0 else cache.v_codes
    s = cache.k_scales if which == 0 else cache.v_scales
    g = cache.k_global if which == 0 else cache.v_global
    assert f32_bits(g[slot].cpu().numpy()) == f32_bits(a32)
    assert np.array_equal(host_u8(c[slot]), codes.reshape(-1))
    assert np.array_equal(host_u8(s[slot]), scales.reshape(-1))
    if smoothed:
        return oracle.kv_dequant_smooth(codes, scales, a32, mean, T, H, d)
    return oracle.kv_dequant(codes, scales, a32, T, H, d)


def _channel_biased(x, seed, scale=2.0):
    """bf16 bits [T, H, d] plus a per-channel offset ~ N(0, scale) (bf16 nearest-even)."""
    T, H, d = x.shape
    g = torch.Generator().manual_seed(seed)
    bias = torch.randn((H, d), generator=g) * scale
    xf = torch.from_numpy(x.astype(np.int32) << 16).view(torch.float32)
    return (xf + bias).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


@pytest.mark.parametrize("smooth_k,smooth_v,search", [(True, False, False), (True, True, True), (False, True, False)])
def test_full_chunk_append_and_dequant_with_smoothing(smooth_k, smooth_v, search):
    """K-smoothing on the workload's 2640 x 24 x 128 chunk (K with per-channel offsets):
    channel means, codes, scales and tensor scales bit for bit, and the bf16 dequant with
    the means added back."""
    require_gpu()
    T, H, d = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    cache = nv.KVCache(3, T, H, d, scale_search=search, smooth_k=smooth_k, smooth_v=smooth_v)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=21)
    k = _channel_biased(k, seed=22)
    cache.append(1, dev_bf16(k), dev_bf16(v))
    slots = torch.tensor([1, 1], dtype=torch.int32, device="cuda")
    ko, vo = cache.dequant(slots)
    torch.cuda.synchronize()
    for which, x, sm, o in ((0, k, smooth_k, ko), (1, v, smooth_v, vo)):
        want = _check_smoothed(cache, 1, x, which, sm, search)
        got = host_bits(o)
        assert np.array_equal(got[0], want) and np.array_equal(got[1], want)


@pytest.mark.parametrize("T,H,d", [(4, 3, 16), (12, 3, 16), (33, 2, 64), (64, 5, 32)])
def test_smoothed_ring_with_ragged_shapes(T, H, d):
    """Smoothed K and V over a ring with a page table, on shapes with fewer tokens than
    partial sums, channel counts that are not a multiple of 64, and short last runs."""
    require_gpu()
    n_slots = 4
    cache = nv.KVCache(n_slots, T, H, d, smooth_k=True, smooth_v=True)
    latest = {}
    for step in range(6):
        k, v = syn.kv_chunk_bf16(T, H, d, seed=300 + step)
        k = _channel_biased(k, seed=400 + step)
        slot = step % n_slots
        cache.append(slot, dev_bf16(k), dev_bf16(v))
        latest[slot] = (k, v)
    order = [2, 3, 0, 1, 3]
    ko, vo = cache.dequant(torch.tensor(order, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    ko, vo = host_bits(ko), host_bits(vo)
    for i, s in enumerate(order):
        for which, x in enumerate(latest[s]):
            want = _check_smoothed(cache, s, x, which, True, False)
            assert np.array_equal((ko if which == 0 else vo)[i], want), (i, s, which)


def test_smoothing_makes_a_channel_constant_chunk_lossless():
    """Every token the same per channel: the smoothed values are 0, so the tensor scale
    is 0, all codes are 0, and the dequant returns the chunk bit for bit."""
    require_gpu()
    T, H, d = 40, 6, 32
    g = np.random.default_rng(5)
    b = (g.integers(-64, 65, size=(H, d)) / 8.0).astype(np.float32)
    x = np.broadcast_to(b, (T, H, d)).copy()
    xb = (x.view(np.uint32) >> 16).astype(np.uint16)
    cache = nv.KVCache(2, T, H, d, smooth_k=True, smooth_v=True)
    cache.append(0, dev_bf16(xb), dev_bf16(xb))
    ko, vo = cache.dequant(torch.tensor([0], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert float(cache.k_global[0]) == 0.0 and float(cache.v_global[0]) == 0.0
    assert not bool(cache.k_codes[0].any()) and not bool(cache.k_scales[0].any())
    assert np.array_equal(host_bits(ko)[0], xb) and np.array_equal(host_bits(vo)[0], xb)


def test_smoothing_reduces_the_error_of_channel_biased_keys():
    """Not parity: on K with per-channel offsets larger than its spread, the smoothed
    store's dequant error is several times smaller than the plain store's."""
    require_gpu()
    T, H, d = 256, 8, 128
    k, v = syn.kv_chunk_bf16(T, H, d, seed=31)
    k = _channel_biased(k, seed=32, scale=8.0)
    slots = torch.tensor([0], dtype=torch.int32, device="cuda")
    errs = []
    for smooth in (False, True):
        cache = nv.KVCache(1, T, H, d, smooth_k=smooth)
        cache.append(0, dev_bf16(k), dev_bf16(v))
        ko, _ = cache.dequant(slots)
        ref = torch.from_numpy(k.astype(np.int32) << 16).view(torch.float32)
        got = ko[0].float().cpu()
        errs.append(float(((got - ref) ** 2).mean()))
    assert errs[1] * 3 < errs[0], errs


def test_dequant_rounds_to_binary32_then_to_bf16():
    """A slot of codes 1.5 with scale 1.0 and a32 = 0.66927087307 (binary32): 1.5 * a32 rounds in binary32 to
    1 + 2^-8, the bf16 midpoint between 1 and 1 + 2^-7, which ties to 1 (0x3F80); a single rounding of the
    exact product would give 0x3F81 (reading R10, two roundings)."""
    require_gpu()
    T, H, d = 4, 1, 16
    a32 = np.float32(0.6692708730697632)
    cache = nv.KVCache(1, T, H, d)
    for t in (cache.k_codes, cache.v_codes):
        t.fill_(0x33)
    for t in (cache.k_scales, cache.v_scales):
        t.fill_(0x38)
    for t in (cache.k_global, cache.v_global):
        t.fill_(float(a32))
    ko, vo = cache.dequant(torch.tensor([0], dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    codes = np.full((T * H, d // 2), 0x33, np.uint8)
    scales = np.full((T * H, d // 16), 0x38, np.uint8)
    want = oracle.kv_dequant(codes, scales, a32, T, H, d)
    assert np.all(want == 0x3F80)
    assert np.array_equal(host_bits(ko)[0], want) and np.array_equal(host_bits(vo)[0], want)
