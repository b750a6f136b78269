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
    """Round finite binary32 values to bf16 (nearest-even) and return the uint16
    bits (32-bit arithmetic: the largest finite pattern plus the rounding
    increment stays below 2^32)."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    return ((u + np.uint32(0x7FFF) + ((u >> np.uint32(16)) & np.uint32(1))) >> np.uint32(16)).astype(np.uint16)


def bf16_bits_to_f32(h: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(h, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def normal_bf16(shape, seed: int, std: float = 1.0) -> np.ndarray:
    g = rng(seed)
    return f32_to_bf16_bits((g.standard_normal(size=shape, dtype=np.float32) * np.float32(std)))


_BLOCK_ROWS = 1024


def normal_bf16_blocks(shape, seed: int, std: float = 1.0, threads: int | None = None) -> np.ndarray:
    """N(0, std^2) bf16 bits [rows, cols] for large tensors: row block i (1024
    rows) is drawn from its own PCG64 stream seeded with (seed, i), blocks in
    parallel threads; the result depends only on (shape, seed, std)."""
    import concurrent.futures as cf
    import os

    rows, cols = shape
    out = np.empty((rows, cols), np.uint16)

    def fill(i):
        r0, r1 = i * _BLOCK_ROWS, min(rows, (i + 1) * _BLOCK_ROWS)
        g = np.random.Generator(np.random.PCG64(np.random.SeedSequence([seed, i])))
        x = g.standard_normal(size=(r1 - r0, cols), dtype=np.float32)
        x *= np.float32(std)
        out[r0:r1] = f32_to_bf16_bits(x)

    n = -(-rows // _BLOCK_ROWS)
    with cf.ThreadPoolExecutor(max_workers=threads or min(32, os.cpu_count() or 1)) as ex:
        list(ex.map(fill, range(n)))
    return out


def stack_layer_bf16(layer: int, D: int = 3072, F: int = 14336):
    """One layer of the DiT linear stack: weights N(0, 0.02) of the QKV
    [3D x D], out-projection [D x D], FFN up [F x D] and FFN down [D x F]
    linears and their N(0, 0.02) biases, as bf16 bits, seeded by the layer."""
    names = (("qkv", 3 * D, D), ("out", D, D), ("up", F, D), ("down", D, F))
    w = {n: normal_bf16_blocks((r, c), seed=10_000 + 8 * layer + i, std=0.02) for i, (n, r, c) in enumerate(names)}
    b = {n: normal_bf16((r,), seed=20_000 + 8 * layer + i, std=0.02) for i, (n, r, _) in enumerate(names)}
    return w, b


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


def rope_table(T: int, d: int, seed: int | None = None, start: int = 0, base: float = 10000.0):
    """A rotary angle table, cos and sin as binary32 [T, d/2]: seeded uniform
    angles in [-pi, pi) when `seed` is given, else token positions start ..
    start + T - 1 times the frequencies base^(-2p/d) (float64, then rounded)."""
    if seed is not None:
        ang = rng(seed).uniform(-np.pi, np.pi, size=(T, d // 2))
    else:
        pos = np.arange(start, start + T, dtype=np.float64)
        ang = pos[:, None] * base ** (-2.0 * np.arange(d // 2, dtype=np.float64) / d)[None, :]
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


def rope_table_3d(frames: int, hh: int, ww: int, d: int, frame0: int = 0, base: float = 10000.0):
    """The 3D (frame, row, column) angle table of a chunk of frames x hh x ww
    latent patches, tokens frame-major: the head's d/2 pairs split into a frame
    band of d/2 - 2*floor(d/6) pairs, then a row band and a column band of
    floor(d/6) pairs each (22, 21, 21 for d = 128); pair i of a band of n pairs
    turns by its axis position times base^(-i/n).  cos and sin as binary32
    [frames*hh*ww, d/2]."""
    npair = d // 2
    nb = d // 6  # pairs per spatial band
    nt = npair - 2 * nb
    f, r, c = np.meshgrid(np.arange(frame0, frame0 + frames), np.arange(hh), np.arange(ww), indexing="ij")
    parts = []
    for pos, n in ((f, nt), (r, nb), (c, nb)):
        freq = base ** (-2.0 * np.arange(n, dtype=np.float64) / (2 * n))
        parts.append(pos.reshape(-1, 1).astype(np.float64) * freq[None, :])
    ang = np.concatenate(parts, axis=1)
    return np.cos(ang).astype(np.float32), np.sin(ang).astype(np.float32)


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
# a chunk's tokens as a latent grid: 3 frames x 22 x 40 patches (720p)
KV_GRID = (3, 22, 40)
