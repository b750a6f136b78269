"""Helpers for the GPU parity tests (test code only)."""
import numpy as np
import pytest
import torch

from bit_video_dit_b200 import build as nvbuild
from bit_video_dit_b200 import nvfp4 as nv


def require_gpu():
    if not torch.cuda.is_available():
        pytest.fail("GPU test run without a CUDA device")
    nvbuild.build()
    nv.lib()


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    """uint16 bf16 bit patterns -> CUDA bf16 tensor (same bits)."""
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16))
    return t.cuda().view(torch.bfloat16)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """CUDA bf16 tensor -> uint16 bit patterns."""
    return t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)


def host_u8(t: torch.Tensor) -> np.ndarray:
    return t.detach().contiguous().cpu().numpy()


def f32_bits(x) -> int:
    return int(np.asarray(x, np.float32).reshape(-1).view(np.uint32)[0])


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def normwise_err(got: np.ndarray, ref: np.ndarray) -> float:
    """max_ij |got - ref| / max_ij |ref| (the GEMM parity metric)."""
    den = float(np.max(np.abs(ref)))
    if den == 0.0:
        return float(np.max(np.abs(got)))
    return float(np.max(np.abs(got - ref))) / den


GEMM_TOL = 2e-3


U32 = 2.0 ** -24  # unit roundoff of binary32


def strided_sum_depth(n: int, group: int = 1) -> int:
    """Most rounded additions any term passes through when n terms (taken in
    groups of `group` consecutive terms) are summed as 32 strided partial sums
    in order, then met in 5 pairwise levels: the order the kernels' headers
    state for the LayerNorm row sums (group 8) and the channel means (group 1)."""
    groups = -(-n // group)
    return group * -(-groups // 32) + 5


def assert_sum_within_bound(got, exact, abs_sum, depth: int, count: int, what: str):
    """A binary32 mean m = fl32(S / count) with S summed at most `depth` deep,
    against the correctly rounded exact mean `exact`: |m - exact| <=
    (depth + 1) u sum|x| / count + 2 u |exact| (the sum's roundings, the
    division's and the reference's own rounding)."""
    got = np.asarray(got, np.float64)
    exact = np.asarray(exact, np.float64)
    bound = (depth + 1) * U32 * np.asarray(abs_sum, np.float64) / count + 2 * U32 * np.abs(exact)
    bad = np.nonzero(np.abs(got - exact) > bound)[0]
    assert bad.size == 0, (f"{what}: {bad.size} values outside the summation bound, first {bad[:4].tolist()}: "
                           f"{got.reshape(-1)[bad[:4]]} vs {exact.reshape(-1)[bad[:4]]}")


def check_ln_stats(stats_dev, x_bits: np.ndarray, eps: float):
    """The kernel's LayerNorm row statistics (binary32 (mean, rstd) per row)
    against the oracle's definition (reading R19) within the binary32 bounds of
    the kernel's stated summation order; returns them (host [rows, 2])."""
    import oracle
    from bit_video_dit_b200 import synthetic as syn

    st = np.ascontiguousarray(stats_dev.detach().cpu().numpy(), np.float32).reshape(-1, 2)
    ref = oracle.ln_stats(x_bits, eps=eps)
    x = syn.bf16_bits_to_f32(x_bits).astype(np.float64)
    rows, cols = x.shape
    depth = strided_sum_depth(cols, 8)
    assert_sum_within_bound(st[:, 0], ref[:, 0], np.abs(x).sum(1), depth, cols, "LayerNorm mean")
    # rstd: the variance's sum has relative error <= (depth + 2) u (a subtraction and a square per
    # term), plus delta^2 / var from the kernel's mean being off by delta; the root, the eps add and
    # the reciprocal each round once more, and the reference's value once
    delta = np.abs(st[:, 0].astype(np.float64) - x.mean(1))
    var = ((x - x.mean(1, keepdims=True)) ** 2).mean(1)
    rel = 0.5 * ((depth + 3) * U32 + delta ** 2 / (var + eps)) + 4 * U32
    r = np.abs(st[:, 1].astype(np.float64) / ref[:, 1].astype(np.float64) - 1.0)
    bad = np.nonzero(r > rel * 1.01)[0]
    assert bad.size == 0, f"LayerNorm rstd: {bad.size} rows outside the bound, first {bad[:4].tolist()}"
    return st


def check_channel_means(mean_dev, values: np.ndarray, ref: np.ndarray, what: str = "channel means"):
    """A kernel's stored binary32 channel means against the oracle's (the
    correctly rounded mean, reading R20) within the bound of the kernel's
    stated order (32 strided partials over the tokens, 5 pairwise levels);
    `values` are the binary32 values averaged, [T, channels...].  Returns the
    kernel's means (host binary32)."""
    m = np.ascontiguousarray(mean_dev.detach().cpu().numpy(), np.float32).reshape(-1)
    v = np.asarray(values, np.float64).reshape(values.shape[0], -1)
    T = v.shape[0]
    assert_sum_within_bound(m, ref.reshape(-1), np.abs(v).sum(0), strided_sum_depth(T), T, what)
    return m
