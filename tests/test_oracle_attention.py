"""Pins of the oracle's attention over the NVFP4 KV cache.

Source: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (reading note), section 二: the
effective KV set of a step is the global sink, the shot-level sink and the window
KV[t - W, t), deduplicated; the KV cache stores each frame-chunk's K and V in NVFP4.
The set is pinned against hand-worked examples (tests/golden/attention_sets.txt); the
fp64 attention against closed forms and torch's scaled_dot_product_attention in
float64 (a library routine), on bf16 inputs.
"""
import os

import numpy as np
import pytest
import torch

import oracle

HERE = os.path.dirname(os.path.abspath(__file__))


def _golden():
    rows = []
    for line in open(os.path.join(HERE, "golden", "attention_sets.txt"), encoding="utf-8"):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        lhs, rhs = line.split(":")
        rows.append((tuple(int(v) for v in lhs.split()), [int(v) for v in rhs.split()]))
    return rows


@pytest.mark.parametrize("args,want", _golden())
def test_attention_chunks_hand_worked(args, want):
    assert oracle.attention_chunks(*args) == want


def bf16(x: np.ndarray) -> np.ndarray:
    b = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return ((b + 0x7FFF + ((b >> 16) & 1)) >> 16).astype(np.uint16)


def f64(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_attention_matches_torch_sdpa_in_float64():
    rng = np.random.default_rng(0)
    Tq, L, H, d = 40, 70, 3, 32
    q, k, v = (bf16(rng.standard_normal((n, H, d)).astype(np.float32)) for n in (Tq, L, L))
    scale = 1.0 / np.sqrt(d)
    got = oracle.attention(q, k, v, scale)
    tq, tk, tv = (torch.from_numpy(f64(x)).permute(1, 0, 2) for x in (q, k, v))
    want = torch.nn.functional.scaled_dot_product_attention(tq, tk, tv, scale=scale).permute(1, 0, 2).numpy()
    assert np.abs(got - want).max() <= 1e-12 * np.abs(want).max()


def test_equal_keys_average_the_values():
    rng = np.random.default_rng(1)
    Tq, L, H, d = 5, 9, 2, 16
    q = bf16(rng.standard_normal((Tq, H, d)).astype(np.float32))
    k = np.broadcast_to(bf16(rng.standard_normal((1, H, d)).astype(np.float32)), (L, H, d)).copy()
    v = bf16(rng.standard_normal((L, H, d)).astype(np.float32))
    got = oracle.attention(q, k, v, 0.3)
    want = np.broadcast_to(f64(v).mean(axis=0), (Tq, H, d))
    assert np.allclose(got, want, rtol=0, atol=1e-12)


def test_a_dominant_key_selects_its_value():
    rng = np.random.default_rng(2)
    Tq, L, H, d = 4, 12, 2, 16
    q = bf16(np.ones((Tq, H, d), np.float32))
    k = bf16(rng.standard_normal((L, H, d)).astype(np.float32) * 0.01)
    k[7] = bf16(np.full((H, d), 8.0, np.float32))
    v = bf16(rng.standard_normal((L, H, d)).astype(np.float32))
    got = oracle.attention(q, k, v, 1.0)
    assert np.allclose(got, np.broadcast_to(f64(v)[7], (Tq, H, d)), rtol=0, atol=1e-12)
