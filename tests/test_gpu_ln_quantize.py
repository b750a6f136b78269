"""GPU parity of nvfp4_ln_modulate_quantize (LayerNorm + adaLN modulate +
NVFP4 quantize, reading R19) against the oracle, in two parts: the kernel's
binary32 row statistics (mean, rstd) against the oracle's definition within
the bounds of the kernel's stated summation order, then codes, scales and the
tensor scale bit for bit against the oracle's modulate + quantize built from
the kernel's own statistics (its binary32 reductions may land a unit away
from the correctly rounded statistics, and the codes follow them)."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import check_ln_stats, dev_bf16, f32_bits, host_u8, require_gpu

pytestmark = pytest.mark.gpu


def _check(x_bits, scale=None, shift=None, *, eps=1e-6, ld=None, alpha=None, rowmajor=False, search=False):
    require_gpu()
    rows, cols = x_bits.shape
    if ld is None:
        xd = dev_bf16(x_bits)
    else:
        buf = np.zeros((rows, ld), np.uint16)
        buf[:, :cols] = x_bits
        xd = dev_bf16(buf)[:, :cols]
    gs = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    ws = nv.workspace(nv.OP_LN_QUANTIZE, rows, 0, cols)
    q = nv.ln_modulate_quantize(xd, mod_scale=None if scale is None else dev_bf16(scale),
                                mod_shift=None if shift is None else dev_bf16(shift), eps=eps, global_scale=gs,
                                rowmajor_scales=rowmajor, scale_search=search, ws=ws)
    torch.cuda.synchronize()
    # the row statistics follow the 256-byte control block of the workspace
    st = check_ln_stats(ws[256:256 + 8 * rows].view(torch.float32), x_bits, eps)
    if search:
        m = oracle.ln_modulate(x_bits, scale, shift, eps=eps, stats=st)
        codes, scales, a32 = oracle.quantize(m, alpha, search46=True)
    else:
        codes, scales, a32 = oracle.ln_modulate_quantize(x_bits, scale, shift, eps=eps, alpha=alpha, stats=st)
    assert f32_bits(q.global_scale.cpu().numpy()) == f32_bits(a32)
    gc = host_u8(q.codes)
    bad = np.argwhere(gc != codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    want = scales.reshape(-1) if rowmajor else oracle.swizzle(scales)
    bad = np.nonzero(host_u8(q.scales) != want)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:4].tolist()}"


def test_dit_activation_full_size():
    """4096 x 3072: each CTA's rows fit in shared memory, so one launch."""
    D = syn.QKV.K
    _check(syn.activations_bf16(4096, D, seed=71), syn.normal_bf16((D,), seed=72, std=0.1),
           syn.normal_bf16((D,), seed=73, std=0.1))


def test_rows_beyond_shared_memory_take_the_two_launch_path():
    """8192 x 3072 (56 rows a CTA, 344 KB): the statistics kernel, then the fused quantize."""
    D = syn.QKV.K
    _check(syn.activations_bf16(8192, D, seed=74), syn.normal_bf16((D,), seed=75, std=0.1),
           syn.normal_bf16((D,), seed=76, std=0.1))


@pytest.mark.parametrize("rows,cols,ld", [(200, 320, None), (129, 576, 640), (1, 64, None), (3, 14336, None)])
def test_ragged_shapes(rows, cols, ld):
    _check(syn.activations_bf16(rows, cols, seed=rows + cols), syn.normal_bf16((cols,), seed=1, std=0.2),
           syn.normal_bf16((cols,), seed=2, std=0.2), ld=ld)


def test_plain_layernorm_given_scale_rowmajor_and_search():
    x = syn.activations_bf16(256, 512, seed=5)
    _check(x)
    _check(x, alpha=0.002)
    _check(x, syn.normal_bf16((512,), seed=6, std=0.1), None, rowmajor=True)
    _check(x, syn.normal_bf16((512,), seed=6, std=0.1), syn.normal_bf16((512,), seed=7, std=0.1), search=True)


def test_constant_rows_and_large_eps():
    x = np.full((64, 128), 0x3FC0, np.uint16)
    x[1::2] = syn.activations_bf16(32, 128, seed=8)
    _check(x, syn.normal_bf16((128,), seed=9, std=0.1), syn.normal_bf16((128,), seed=10, std=0.1), eps=0.5)
