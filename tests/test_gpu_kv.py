"""GPU parity of the NVFP4 KV-cache store: nvfp4_kv_append (codes, row-major
scales and per-slot tensor scales bit for bit) and nvfp4_kv_dequant (bf16 bit
for bit), on the workload's 2640 x 24 x 128 chunk and on small rings."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import dev_bf16, f32_bits, host_bits, host_u8, require_gpu

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
