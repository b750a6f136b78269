"""GPU check of nvfp4_quantize_noalloc, the quantize entry point for callers
that cannot allocate device memory (code inside a framework that owns every
device allocation, or a loop that must not call cudaMalloc).  It must give
exactly what nvfp4_quantize gives with a caller workspace, and it must do so
on consecutive calls, since every call reuses the same static scratch.

This file is named to be collected last, so a failure here comes after every
other test has run.
"""

import numpy as np
import pytest
import torch

from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import dev_bf16, require_gpu

pytestmark = pytest.mark.gpu


def _noalloc(x: torch.Tensor, alpha=None) -> nv.NVFP4Tensor:
    rows, cols = x.shape
    out = nv.empty_nvfp4(rows, cols, x.device)
    flags = nv.Q_COMPUTE_GLOBAL
    if alpha is not None:
        out.global_scale.fill_(float(alpha))
        flags = nv.Q_GIVEN_GLOBAL
    st = nv.lib().nvfp4_quantize_noalloc(x.data_ptr(), rows, cols, x.stride(0), out.codes.data_ptr(),
                                         out.scales.data_ptr(), out.global_scale.data_ptr(), flags,
                                         torch.cuda.current_stream().cuda_stream)
    assert st == nv.OK, nv.status_string(st)
    return out


def _same(a: nv.NVFP4Tensor, b: nv.NVFP4Tensor):
    torch.cuda.synchronize()
    assert torch.equal(a.codes, b.codes)
    assert torch.equal(a.scales, b.scales)
    assert a.global_scale.view(torch.int32).item() == b.global_scale.view(torch.int32).item()


def test_noalloc_matches_workspace_quantize_on_consecutive_calls():
    require_gpu()
    x1 = dev_bf16(syn.activations_bf16(4096, 3072, seed=2))
    x2 = dev_bf16(syn.activations_bf16(200, 320, seed=77))
    # two calls in a row on different inputs, each against the workspace path
    _same(_noalloc(x1), nv.quantize(x1))
    _same(_noalloc(x2), nv.quantize(x2))
    # and once more with a given tensor scale
    a = 0.5 * float(nv.quantize(x2).global_scale.item())
    _same(_noalloc(x2, alpha=a), nv.quantize(x2, global_scale=torch.tensor([a], device="cuda")))


def test_noalloc_rejects_bad_arguments_on_the_host():
    require_gpu()
    L = nv.lib()
    assert L.nvfp4_quantize_noalloc(None, 16, 48, 48, None, None, None, 0, None) in (nv.ERR_INVALID_ARG,
                                                                                      nv.ERR_UNSUPPORTED)
    assert L.nvfp4_quantize_noalloc(None, -1, 64, 64, None, None, None, 0, None) == nv.ERR_INVALID_ARG
