"""Seeded synthetic inputs shared by the tests, the smoke check and the bench.

This module draws random numbers and rounds them to bf16 bit patterns; it holds
none of the NVFP4 arithmetic.  Both the CUDA path and the CPU oracle consume the
exact same bf16 buffers produced here.

Shapes follow the DiT linear and KV shapes of a Wan2.2-TI2V-5B-sized model
(hidden 3072, FFN 14336, 24 heads x 128), as used by LongLive-2.0
("LongLive-2.0：用 NVFP4 并行底座做长视频生成", yingwang.github.io reading note,
section 三 实验).  Activations are N(0,1) with a few outlier channels scaled
x20 (LLM/DiT activations carry such channels; the pages' own inputs are video
latents that are not available here), weights N(0, 0.02).
"""
from __future__ import annotations

from dataclasses import dataclass

import numpy as np


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round binary32 values to bf16 (nearest-even) and return the uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32).astype(np.uint64)
    r = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return r.astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    g = rng(seed)
    return f32_to_bf16_bits((g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)))


def activations_bf16(rows: int, cols: int, seed: int, outlier_frac: float = 0.001,
                     outlier_scale: float = 20.0) -> np.ndarray:
    """N(0,1) activations with floor(outlier_frac*cols) (at least 1) outlier
    channels (columns) scaled by outlier_scale; channel choice is seeded."""
    g = rng(seed)
    x = g.standard_normal(size=(rows, cols), dtype=np.float32)
    n_out = max(1, int(np.floor(outlier_frac * cols)))
    ch = g.choice(cols, size=n_out, replace=False)
    x[:, ch] *= np.float32(outlier_scale)
    return f32_to_bf16_bits(x)


def tiny_a_bf16(rows: int = 64, cols: int = 256, seed: int = 0, frac: float = 0.01,
                scale: float = 30.0) -> np.ndarray:
    """N(0,1) with round(frac*rows*cols) entries (uniform, without replacement) x scale."""
    g = rng(seed)
    x = g.standard_normal(size=(rows, cols), dtype=np.float32)
    n = int(round(frac * rows * cols))
    idx = g.choice(rows * cols, size=n, replace=False)
    x.reshape(-1)[idx] *= np.float32(scale)
    return f32_to_bf16_bits(x)


def kv_chunk_bf16(T: int, H: int, d: int, seed: int):
    """One frame-chunk's K and V, token-major [T, H, d], N(0,1) with every head
    scaled by its own c_h ~ U(0.5, 4) (drawn per head for K and for V)."""
    g = rng(seed)
    out = []
    for _ in range(2):
        x = g.standard_normal(size=(T, H, d), dtype=np.float32)
        c = g.uniform(0.5, 4.0, size=(H,)).astype(np.float32)
        x *= c[None, :, None]
        out.append(f32_to_bf16_bits(x))
    return out[0], out[1]


@dataclass(frozen=True)
class GemmShape:
    M: int
    N: int
    K: int


# The linear-layer shapes of the workloads (tokens x out-features x in-features).
TINY = GemmShape(64, 128, 256)
QKV = GemmShape(4096, 9216, 3072)
FFN_UP = GemmShape(8192, 14336, 3072)
FFN_DOWN = GemmShape(8192, 3072, 14336)
STACK_M = 16384
STACK_LAYERS = 30
STACK_LAYER = (GemmShape(STACK_M, 9216, 3072), GemmShape(STACK_M, 3072, 3072),
               GemmShape(STACK_M, 14336, 3072), GemmShape(STACK_M, 3072, 14336))

# NVFP4 KV cache: 21 ring slots (frame-chunks) x 2640 tokens x 24 heads x 128.
KV_SLOTS, KV_TOKENS, KV_HEADS, KV_DIM = 21, 2640, 24, 128
