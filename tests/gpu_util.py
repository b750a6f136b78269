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
