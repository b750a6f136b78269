"""GPU parity of nvfp4_kv_attention (softmax attention of bf16 queries over NVFP4
cache slots read directly by the kernel) against the oracle's fp64 attention over
the same slots' values -- exact e2m1 * s * a32 for a cache without smoothing, the
bf16 dequant with the means otherwise (reading R23: max |O - O_ref| / max |O_ref|
<= 1e-2)."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import dev_bf16, host_bits, normwise_err, require_gpu

pytestmark = pytest.mark.gpu
TOL = 1e-2


def _bits_to_f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _case(T, H, Tq, slot_chunks, n_slots, seed, smooth_k=False, smooth_v=False, scale=0.0, rows=None):
    """Fill a cache with seeded chunks, attend with seeded queries over the listed slots;
    compare against the oracle (on sampled query rows when `rows` is given)."""
    d = 128
    cache = nv.KVCache(n_slots, T, H, d, smooth_k=smooth_k, smooth_v=smooth_v)
    # keys and values as the kernel reads them (reading R23): without smoothing the cache's
    # exact values e2m1 * s * a32 (binary16 path); with smoothing on either tensor the
    # cache's bf16 dequant (plus the means) for both
    raw = not (smooth_k or smooth_v)
    kh, vh, av = {}, {}, {}
    for s in range(n_slots):
        k, v = syn.kv_chunk_bf16(T, H, d, seed=seed + s)
        cache.append(s, dev_bf16(k), dev_bf16(v))
        for name, x, sm, store in (("k", k, smooth_k, kh), ("v", v, smooth_v, vh)):
            if sm:
                # the codes follow the kernel's stored means (checked against the oracle's
                # within their summation bound in the KV tests)
                km = (cache.k_mean if name == "k" else cache.v_mean)[s].cpu().numpy()
                c, sc, a, m = oracle.kv_append_smooth(x, mean=km)
                store[s] = oracle.kv_dequant_smooth(c, sc, a, m, T, H, d)
            else:
                c, sc, a = oracle.kv_append(x)
                store[s] = (oracle.dequant_f32(c, sc, a).reshape(T, H, d) if raw
                            else oracle.kv_dequant(c, sc, a, T, H, d))
                if name == "v":
                    av[s] = float(a)
    q = syn.kv_chunk_bf16(Tq, H, d, seed=seed + 1000)[0]
    slots = torch.tensor(slot_chunks, dtype=torch.int32, device="cuda")
    o = cache.attention(slots, dev_bf16(q), scale=scale)
    torch.cuda.synchronize()
    got = _bits_to_f64(host_bits(o))
    if not slot_chunks:
        return got, None, cache
    kk = np.concatenate([kh[s] for s in slot_chunks], axis=0)
    vv = np.concatenate([vh[s] for s in slot_chunks], axis=0)
    sc = scale if scale > 0 else 1.0 / np.sqrt(d)
    qs = q if rows is None else q[rows]
    ref = oracle.attention(qs, kk, vv, sc)
    gs = got if rows is None else got[rows]
    err = normwise_err(gs.reshape(-1), ref.reshape(-1))
    assert err <= TOL, err
    # binary16 path: each key's P carries its slot's a32_V / a32_ref
    w = None
    if raw:
        a_ref = max(av[s] for s in slot_chunks)
        w = np.concatenate([np.full(T, av[s] / a_ref if a_ref > 0 else 0.0) for s in slot_chunks])
    check_rows(gs, qs, kk, vv, sc, ref, w)
    return got, ref, cache


def check_rows(got, q, k, v, scale, ref, w=None):
    """Per element of every output row (reading R23's error sources): P rounded
    to its 16-bit type moves each weight by at most 2^-11 of itself while it is
    in binary16's normal range, so the numerator by at most 2^-11 of
    sum_j p_j |v_j|; O's bf16 store and the binary32 row sum add at most ~2^-9
    |O|.  A binary16 weight below the normal range (2^-14) is off by up to
    2^-25 absolute instead; the row's weights are relative to a reference at
    or below its largest score, so at most the keys whose weight relative to
    that score, times the slot's V weight w = a32_V / a32_ref, is below 2^-14
    are subnormal, each adding 2^-25 a32_ref |e2m1 s| / l = 2^-25 |V_j| / (w_j l)
    (l = the row's weight sum, >= 1).  Bound, with room:
      |O - O_ref| <= 2^-8 (softmax-weighted |V|) + 2^-8 |O_ref| + 2^-25 max_j(|V_j| / w_j) n_sub / l."""
    vf = _bits_to_f64(v) if v.dtype == np.uint16 else np.asarray(v, np.float64)
    qf = _bits_to_f64(q) if q.dtype == np.uint16 else np.asarray(q, np.float64)
    wabs = oracle.attention(q, k, np.abs(vf), scale)
    ww = np.ones(k.shape[0]) if w is None else np.asarray(w, np.float64)
    # per head, the largest binary16 operand value times a32_ref: max_j |V_j| / w_j (a slot with w = 0
    # holds zeros)
    vk = np.abs(vf).max(axis=2)
    cap = np.where(ww[:, None] > 0, vk / np.where(ww[:, None] > 0, ww[:, None], 1.0), 0.0).max(axis=0)
    sub = np.zeros(ref.shape[:2])
    for h in range(ref.shape[1]):
        kh = _bits_to_f64(k[:, h, :]) if k.dtype == np.uint16 else np.asarray(k[:, h, :], np.float64)
        t = (qf[:, h, :] @ kh.T) * scale
        p = np.exp(t - t.max(axis=1, keepdims=True))
        sub[:, h] = 2.0 ** -25 * cap[h] * np.sum(p * ww[None, :] < 2.0 ** -14, axis=1) / p.sum(axis=1)
    bound = 2.0 ** -8 * wabs + 2.0 ** -8 * np.abs(ref) + sub[:, :, None]
    excess = np.abs(got - ref) - bound
    worst = np.unravel_index(np.argmax(excess), excess.shape)
    assert np.all(excess <= 0), (f"row element outside the bound at {worst}: got {got[worst]} ref {ref[worst]} "
                                 f"bound {bound[worst]}")


@pytest.mark.parametrize("T,Tq", [(256, 200), (200, 128), (130, 7)])
def test_small_sets_with_ragged_tiles(T, Tq):
    require_gpu()
    _case(T, 2, Tq, [0, 2], 3, seed=40 + T)


def test_sink_and_window_set_from_the_chunk_builder():
    """Step t = 9 of a ring of 6 slots: global sink 1, shot sink 1 (shot from chunk 4), window 3;
    chunk c lives in slot c mod 6 except the pinned sink in slot 0."""
    require_gpu()
    chunks = nv.attention_chunks(9, 1, 4, 1, 3)
    assert chunks == [0, 4, 6, 7, 8]
    slots = [0 if c == 0 else 1 + (c - 1) % 5 for c in chunks]
    _case(160, 3, 150, slots, 6, seed=60)


@pytest.mark.parametrize("smooth_k,smooth_v", [(True, False), (True, True)])
def test_smoothed_cache(smooth_k, smooth_v):
    require_gpu()
    _case(192, 2, 140, [1, 0], 2, seed=80, smooth_k=smooth_k, smooth_v=smooth_v)


def test_given_scale_and_repeated_slot():
    require_gpu()
    _case(128, 2, 64, [1, 1, 0], 2, seed=90, scale=0.05)


def test_full_chunk_workload_on_sampled_queries():
    """The KV workload's chunk (2640 tokens x 24 heads x 128) attending over three slots
    (a sink and a two-chunk window) with a full 2640-token query chunk; 48 sampled rows."""
    require_gpu()
    rows = np.sort(np.random.default_rng(7).choice(2640, 48, replace=False))
    _case(syn.KV_TOKENS, syn.KV_HEADS, syn.KV_TOKENS, [0, 2, 3], 4, seed=100, rows=rows)


def test_empty_list_gives_zeros_and_bad_slot_is_reported():
    require_gpu()
    got, _, _ = _case(128, 2, 32, [], 2, seed=110)
    assert not np.any(got)
    T, H, d = 128, 2, 128
    cache = nv.KVCache(2, T, H, d)
    k, v = syn.kv_chunk_bf16(T, H, d, seed=111)
    cache.append(0, dev_bf16(k), dev_bf16(v))
    q = dev_bf16(syn.kv_chunk_bf16(16, H, d, seed=112)[0])
    ws = nv.workspace(nv.OP_KV_ATTENTION, device="cuda")
    cache.attention(torch.tensor([0, 5], dtype=torch.int32, device="cuda"), q, ws=ws)
    code, info = nv.read_device_error(ws)
    assert code == nv.ERR_DEVICE and info == 1


def test_smoothed_channel_constant_slot_with_zero_tensor_scale():
    """A smoothed K chunk that is constant per channel has tensor scale 0 and all codes 0;
    its keys are the means, which the attention must still add."""
    require_gpu()
    T, H, d = 96, 2, 128
    cache = nv.KVCache(1, T, H, d, smooth_k=True)
    rng = np.random.default_rng(3)
    b = (rng.integers(-16, 17, size=(H, d)) / 8.0).astype(np.float32)
    kb = (np.broadcast_to(b, (T, H, d)).copy().view(np.uint32) >> 16).astype(np.uint16)
    _, v = syn.kv_chunk_bf16(T, H, d, seed=5)
    cache.append(0, dev_bf16(kb), dev_bf16(v))
    assert float(cache.k_global[0]) == 0.0
    q = syn.kv_chunk_bf16(40, H, d, seed=6)[0]
    o = cache.attention(torch.tensor([0], dtype=torch.int32, device="cuda"), dev_bf16(q))
    torch.cuda.synchronize()
    c, sc, a = oracle.kv_append(v)  # smoothed cache: the bf16 path for both tensors
    ref = oracle.attention(q, kb, oracle.kv_dequant(c, sc, a, T, H, d), 1.0 / np.sqrt(d))
    assert normwise_err(_bits_to_f64(host_bits(o)).reshape(-1), ref.reshape(-1)) <= TOL


def test_lazy_maximum_rescale_is_forced_and_counted():
    """Even query rows align with one late key (token 300 of a 384-token slot, in the
    third key tile) whose score exceeds every earlier one by far more than 2^8 in the
    exponent, so those rows move their reference maximum and O is rescaled in TMEM;
    odd rows of the same warps do not (they multiply by exactly 1).  The workspace's
    rescale counter records it, and O matches the oracle per element."""
    require_gpu()
    T, H, d, Tq = 384, 2, 128, 128
    rng = np.random.default_rng(17)
    kf = (rng.standard_normal((T, H, d)) * 0.1).astype(np.float32)
    kf[300] = 0.5
    vf = rng.standard_normal((T, H, d)).astype(np.float32)
    qf = (rng.standard_normal((Tq, H, d)) * 0.3).astype(np.float32)
    qf[0::2] = 2.0
    kb, vb, qb = (syn.f32_to_bf16_bits(x) for x in (kf, vf, qf))
    cache = nv.KVCache(1, T, H, d)
    cache.append(0, dev_bf16(kb), dev_bf16(vb))
    ws = nv.workspace(nv.OP_KV_ATTENTION, device="cuda")
    o = cache.attention(torch.tensor([0], dtype=torch.int32, device="cuda"), dev_bf16(qb), ws=ws)
    torch.cuda.synchronize()
    rescales = int(ws[16:20].view(torch.int32).item())
    # 1 query tile x 2 heads x 4 warps, each with even rows that move at the third key tile
    assert rescales >= 8, rescales
    kc, ksc, ka = oracle.kv_append(kb)
    vc, vsc, va = oracle.kv_append(vb)
    kk = oracle.dequant_f32(kc, ksc, ka).reshape(T, H, d)
    vv = oracle.dequant_f32(vc, vsc, va).reshape(T, H, d)
    sc = 1.0 / np.sqrt(d)
    ref = oracle.attention(qb, kk, vv, sc)
    got = _bits_to_f64(host_bits(o))
    assert normwise_err(got.reshape(-1), ref.reshape(-1)) <= TOL
    check_rows(got, qb, kk, vv, sc, ref)
    # the even rows are dominated by value row 300 (the rescale really mattered)
    assert np.allclose(ref[0::2], vv[300][None].astype(np.float64), rtol=0, atol=5e-2 * np.abs(vv[300]).max())


def test_twenty_one_slot_workload_set_on_sampled_rows():
    """The bench's attention: one 2640 x 24 x 128 query chunk over all 21 ring slots
    (55,440 keys per head) of the KV workload's cache, checked on 32 sampled query rows
    normwise and per element."""
    require_gpu()
    rows = np.sort(np.random.default_rng(21).choice(syn.KV_TOKENS, 32, replace=False))
    _case(syn.KV_TOKENS, syn.KV_HEADS, syn.KV_TOKENS, list(range(syn.KV_SLOTS)), syn.KV_SLOTS, seed=200, rows=rows)


def test_zero_value_slot_in_the_binary16_path():
    """A cache without smoothing where one listed slot's V chunk is all zero (tensor scale
    0, so its P weights are stored as exactly 0) while its keys still take part in every
    row's sum: O matches the oracle normwise and per element."""
    require_gpu()
    T, H, d, Tq = 200, 2, 128, 150
    cache = nv.KVCache(3, T, H, d)
    kh, vh, av = {}, {}, {}
    for s in range(3):
        k, v = syn.kv_chunk_bf16(T, H, d, seed=300 + s)
        if s == 1:
            v = np.zeros_like(v)
        cache.append(s, dev_bf16(k), dev_bf16(v))
        for x, store in ((k, kh), (v, vh)):
            c, sc, a = oracle.kv_append(x)
            store[s] = oracle.dequant_f32(c, sc, a).reshape(T, H, d)
        av[s] = float(a)
    assert float(cache.v_global[1]) == 0.0
    q = syn.kv_chunk_bf16(Tq, H, d, seed=310)[0]
    listed = [0, 1, 2]
    o = cache.attention(torch.tensor(listed, dtype=torch.int32, device="cuda"), dev_bf16(q))
    torch.cuda.synchronize()
    kk = np.concatenate([kh[s] for s in listed], axis=0)
    vv = np.concatenate([vh[s] for s in listed], axis=0)
    sc = 1.0 / np.sqrt(d)
    ref = oracle.attention(q, kk, vv, sc)
    got = _bits_to_f64(host_bits(o))
    assert normwise_err(got.reshape(-1), ref.reshape(-1)) <= TOL
    a_ref = max(av.values())
    w = np.concatenate([np.full(T, av[s] / a_ref) for s in listed])
    check_rows(got, q, kk, vv, sc, ref, w)


def test_large_scale_spreads_the_scores():
    """scale = 1 (instead of 1/sqrt(d)) spreads each row's scores over tens of binary
    exponents, so rows move their reference maximum across tiles and slots and many
    weights fall far below the maximum; O still matches the oracle per element."""
    require_gpu()
    _case(384, 2, 200, [0, 1, 2], 3, seed=320, scale=1.0)
