"""GPU parity of nvfp4_quantize against the CPU oracle: codes, scales (swizzled
bytes including the zero padding) and the tensor scale, bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn

from .gpu_util import dev_bf16, f32_bits, host_u8, require_gpu

pytestmark = pytest.mark.gpu


def _check(x_bits, *, ld=None, alpha=None, rowmajor=False, search=False):
    require_gpu()
    rows, cols = x_bits.shape
    if ld is None:
        xd = dev_bf16(x_bits)
    else:  # embed in a wider buffer: row stride ld elements
        buf = np.zeros((rows, ld), np.uint16)
        buf[:, :cols] = x_bits
        xd = dev_bf16(buf)[:, :cols]
    gs = None if alpha is None else torch.tensor([alpha], dtype=torch.float32, device="cuda")
    q = nv.quantize(xd, global_scale=gs, rowmajor_scales=rowmajor, scale_search=search)
    torch.cuda.synchronize()
    codes, scales, a32 = oracle.quantize(x_bits, alpha, search46=search)
    assert f32_bits(q.global_scale.cpu().numpy()) == f32_bits(a32)
    gc = host_u8(q.codes)
    bad = np.argwhere(gc != codes)
    assert bad.size == 0, f"{len(bad)} code bytes differ, first at {bad[:4].tolist()}"
    gsc = host_u8(q.scales)
    want = scales.reshape(-1) if rowmajor else oracle.swizzle(scales)
    assert gsc.shape == want.shape
    bad = np.nonzero(gsc != want)[0]
    assert bad.size == 0, f"{bad.size} scale bytes differ, first at {bad[:4].tolist()}"
    return q


def test_tiny_operands():
    _check(syn.tiny_a_bf16(64, 256, seed=0))
    _check(syn.normal_bf16((128, 256), seed=1))


def test_qkv_activation_full_size():
    _check(syn.activations_bf16(4096, 3072, seed=2))


def test_qkv_weight_full_size():
    _check(syn.normal_bf16((9216, 3072), seed=3, std=0.02))


@pytest.mark.parametrize("rows,cols,ld", [(1, 64, None), (200, 320, None), (129, 576, 640), (3, 1024, None),
                                          (130, 64, 72), (257, 128, None)])
def test_ragged_shapes_and_strides(rows, cols, ld):
    _check(syn.activations_bf16(rows, cols, seed=rows + cols), ld=ld)


@pytest.mark.parametrize("search,rowmajor", [(False, True), (True, False)])
def test_inputs_beyond_shared_memory_take_the_register_kernel(search, rowmajor):
    """8192 x 3072 (25 M elements) is past what the staged kernel holds in shared memory
    (~17 M per launch): the fused kernel, which holds part of the runs in registers and
    reads the rest again for the encode."""
    _check(syn.activations_bf16(8192, 3072, seed=9), search=search, rowmajor=rowmajor)


def test_back_to_back_launches_on_one_workspace():
    """Twenty quantizes of different inputs queued on one stream with one workspace, no synchronisation between
    them: the grid barrier's words alternate by launch parity and each launch resets the other parity's, so every
    tensor scale and code comes out as the oracle's (a barrier word left over from a previous launch would merge
    two launches' maxima)."""
    require_gpu()
    xs = [syn.activations_bf16(256 + 64 * (i % 3), 512, seed=300 + i) for i in range(20)]
    # the third input is all zero: its tensor scale must not inherit a neighbour's maximum
    xs[2] = np.zeros_like(xs[2])
    ws = nv.workspace(nv.OP_QUANTIZE, 384, 0, 512)
    xd = [dev_bf16(x) for x in xs]
    torch.cuda.synchronize()
    outs = [nv.quantize(d, ws=ws) for d in xd]
    torch.cuda.synchronize()
    for x, q in zip(xs, outs):
        codes, scales, a32 = oracle.quantize(x)
        assert f32_bits(q.global_scale.cpu().numpy()) == f32_bits(a32)
        assert np.array_equal(host_u8(q.codes), codes)
        assert np.array_equal(host_u8(q.scales), oracle.swizzle(scales))


def test_all_zero_tensor():
    q = _check(np.zeros((64, 128), np.uint16))
    assert float(q.global_scale.item()) == 0.0


def test_given_scale_saturates_and_flushes():
    x = syn.activations_bf16(128, 512, seed=7)
    _, _, a32 = oracle.quantize(x)
    _check(x, alpha=np.float32(a32 / 8))    # block scales saturate at 448
    _check(x, alpha=np.float32(a32 * 1e5))  # most block scales flush to zero


def test_rowmajor_scales():
    _check(syn.activations_bf16(96, 256, seed=8), rowmajor=True)


def test_zero_rows_is_a_noop():
    require_gpu()
    x = torch.empty((0, 64), dtype=torch.bfloat16, device="cuda")
    q = nv.quantize(x)
    assert q.codes.numel() == 0


# ---- adaptive scale search over the targets {4, 6} (NVFP4_Q_SCALE_SEARCH) ----

def test_scale_search_activation_full_size():
    q = _check(syn.activations_bf16(4096, 3072, seed=2), search=True)
    # it does pick the target-4 encoding for part of the blocks
    std = nv.quantize(dev_bf16(syn.activations_bf16(4096, 3072, seed=2)))
    torch.cuda.synchronize()
    frac = (q.scales != std.scales).float().mean().item()
    assert 0.01 < frac < 0.99


@pytest.mark.parametrize("rows,cols,ld,rowmajor", [(200, 320, None, False), (129, 576, 640, True), (1, 64, None, False)])
def test_scale_search_ragged(rows, cols, ld, rowmajor):
    _check(syn.activations_bf16(rows, cols, seed=rows * 7 + cols), ld=ld, rowmajor=rowmajor, search=True)


def test_scale_search_given_scale_and_zero_tensor():
    x = syn.normal_bf16((128, 256), seed=5)
    _check(x, alpha=0.01, search=True)
    _check(np.zeros((64, 128), np.uint16), search=True)


def test_rounding_boundary_blocks():
    """The blocks the oracle pins on rounding boundaries (given a32 = 1), with and without the scale search: an
    element on an E2M1 midpoint where the binary32 reciprocal of s * a32 and a division disagree (R5), sixteen
    6.0 that both search targets represent exactly (a tie keeps the standard encoding, R18), and blocks exact
    under one target only."""
    xf = np.zeros((4, 64), np.float32)
    xf[0, 0], xf[0, 1] = 0.17578125, 0.0732421875
    xf[1, 0:16] = 6.0
    xf[2, 0:16] = [4, 3, 2, 1.5, 1, 0.5, 0, -4, -3, -2, -1.5, -1, -0.5, 4, 2, 1]
    xf[3, 0:16] = [6, 3, 1.5, 0.5, 0, -6, 2, 1, -0.5, 4, -3, 1.5, 0, 0, 6, -1]
    x = syn.f32_to_bf16_bits(xf)
    for search in (False, True):
        _check(x, alpha=1.0, search=search)
