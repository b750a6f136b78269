"""CPU checks of the C-ABI boundary: libnvfp4.so loads without a GPU, exports
every function include/nvfp4.h declares, answers the size queries, and rejects
bad arguments on the host before touching the device."""
import ctypes
import os
import re

import pytest

from bit_video_dit_b200 import build as nvbuild
from bit_video_dit_b200 import nvfp4 as nv

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def L():
    nvbuild.build()
    return nv.lib()


def _declared_functions():
    text = open(os.path.join(ROOT, "include", "nvfp4.h")).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(nvfp4_[a-z0-9_]+)\s*\(", text)))


def test_every_declared_function_is_exported(L):
    names = _declared_functions()
    assert len(names) >= 10
    for n in names:
        assert hasattr(L, n), n
    assert set(names) == set(nv.EXPORTS)


def test_size_queries(L):
    assert nv.codes_bytes(4096, 3072) == 4096 * 1536
    assert nv.scales_bytes(4096, 3072, True) == 4096 * 192
    assert nv.scales_bytes(4096, 3072, False) == 4096 * 192
    assert nv.scales_bytes(200, 320, True) == 256 * 20
    assert nv.scales_bytes(1, 64, True) == 128 * 4
    assert nv.codes_bytes(3, 5) == 0 and nv.scales_bytes(3, 8, True) == 0
    for op in range(4):
        assert nv.workspace_bytes(op, 4096, 9216, 3072) >= 16
    assert nv.status_string(nv.OK) == "ok"
    assert "wait" in nv.status_string(nv.ERR_TIMEOUT)
    assert L.nvfp4_version() >> 16 == 1


def test_kv_bytes_are_nine_eighths(L):
    # K + V per chunk: 2 * (codes + row-major scales) = 9/8 * T * H * d
    T, H, d = 2640, 24, 128
    per = nv.codes_bytes(T * H, d) + nv.scales_bytes(T * H, d, False)
    assert 2 * per == 9 * T * H * d // 8


def test_host_side_argument_checks(L):
    st = L.nvfp4_quantize(None, 16, 64, 64, None, None, None, 0, None, 0, None)
    assert st == nv.ERR_INVALID_ARG
    fake = 1 << 20  # never dereferenced: the checks below fail first
    st = L.nvfp4_quantize(fake, 16, 48, 48, fake, fake, fake, 0, fake, 1 << 16, None)
    assert st == nv.ERR_UNSUPPORTED  # cols % 64 != 0
    st = L.nvfp4_quantize(fake, 16, 64, 64, fake, fake, fake, 8, fake, 1 << 16, None)
    assert st == nv.ERR_INVALID_ARG  # unknown flag
    st = L.nvfp4_quantize(fake + 8, 16, 64, 64, fake, fake, fake, 0, fake, 1 << 16, None)
    assert st == nv.ERR_MISALIGNED
    st = L.nvfp4_quantize(fake, 16, 64, 64, fake, fake, fake, 0, fake, 16, None)
    assert st == nv.ERR_INVALID_ARG  # workspace too small
    # the no-allocation quantize runs the same checks before touching its shared scratch (here,
    # with no GPU, any CUDA call would fail with NVFP4_ERR_CUDA instead)
    nq = L.nvfp4_quantize_noalloc
    assert nq(fake, 16, 48, 48, fake, fake, fake, 0, None) == nv.ERR_UNSUPPORTED  # cols % 64
    assert nq(fake, 16, 64, 64, fake, fake, fake, 8, None) == nv.ERR_INVALID_ARG  # unknown flag
    assert nq(fake + 8, 16, 64, 64, fake, fake, fake, 0, None) == nv.ERR_MISALIGNED
    assert nq(fake, 16, 64, 64, fake, fake, None, 0, None) == nv.ERR_INVALID_ARG  # no tensor scale
    assert nq(fake, 0, 64, 64, fake, fake, fake, 0, None) == nv.OK  # nothing to do, nothing enqueued
    a = nv.CTensor(fake, fake, fake, 64, 256)
    b = nv.CTensor(fake, fake, fake, 128, 192)
    st = L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), fake, 128, None, fake, 4096, None)
    assert st == nv.ERR_INVALID_ARG  # K mismatch
    b = nv.CTensor(fake, fake, fake, 128, 96)
    a = nv.CTensor(fake, fake, fake, 64, 96)
    st = L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), fake, 128, None, fake, 4096, None)
    assert st == nv.ERR_UNSUPPORTED  # K % 64
    a = nv.CTensor(fake, fake, fake, 64, 256)
    b = nv.CTensor(fake, fake, fake, 128, 256)
    st = L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), None, 128, None, fake, 4096, None)
    assert st == nv.ERR_INVALID_ARG  # no output at all
    st = L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), fake + 16, 100, None, fake, 4096, None)
    assert st == nv.ERR_INVALID_ARG  # ldc < N
    # the requant / out_amax column window: inside [0, N), multiples of 64 for a requant
    b = nv.CTensor(fake, fake, fake, 512, 256)
    for window, want in (((64, 0), nv.OK), ((96, 64), nv.ERR_UNSUPPORTED), ((64, 96), nv.ERR_UNSUPPORTED),
                         ((448, 128), nv.ERR_INVALID_ARG), ((-64, 64), nv.ERR_INVALID_ARG),
                         ((512, 0), nv.ERR_INVALID_ARG)):
        ep = nv.CEpilogue(out_codes=fake, out_scales=fake, out_global_scale=fake, out_col0=window[0],
                          out_cols=window[1], ld_residual=0, act=9)  # act 9: rejected after the window checks
        st = L.nvfp4_gemm(ctypes.byref(a), ctypes.byref(b), None, 512, ctypes.byref(ep), fake, 4096, None)
        assert st == (nv.ERR_INVALID_ARG if want == nv.OK else want), window
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 24)
    st = L.nvfp4_kv_append(ctypes.byref(kv), 0, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_UNSUPPORTED  # head_dim % 16
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 32)
    st = L.nvfp4_kv_append(ctypes.byref(kv), 4, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_INVALID_ARG  # slot out of range
    st = L.nvfp4_kv_dequant(ctypes.byref(kv), fake, -1, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_INVALID_ARG
    # K-smoothing: the flagged tensor's mean array is required and 16-byte aligned
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 32, nv.KV_SMOOTH_K)
    st = L.nvfp4_kv_append(ctypes.byref(kv), 0, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_INVALID_ARG  # no k_mean
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 32, nv.KV_SMOOTH_V, fake, fake + 4)
    st = L.nvfp4_kv_dequant(ctypes.byref(kv), fake, 1, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_MISALIGNED  # v_mean not 16-byte aligned
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 1 << 24, 1, 16, nv.KV_SMOOTH_K, fake, fake)
    st = L.nvfp4_kv_append(ctypes.byref(kv), 0, fake, fake, fake, 1 << 30, None)
    assert st == nv.ERR_UNSUPPORTED  # T = 2^24 tokens: not exact as a binary32 divisor
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 32, 8)
    st = L.nvfp4_kv_append(ctypes.byref(kv), 0, fake, fake, fake, 1 << 16, None)
    assert st == nv.ERR_INVALID_ARG  # unknown flag
    # rows longer than 2^30 elements (a KV chunk is one row of T*H*d) are refused before any launch
    st = L.nvfp4_quantize(fake, 1, (1 << 30) + 64, (1 << 30) + 64, fake, fake, fake, 0, fake, 1 << 16, None)
    assert st == nv.ERR_UNSUPPORTED
    # so are tensors of 2^31 or more 16-element blocks (the kernel's block index is 32 bits)
    st = L.nvfp4_quantize(fake, 1 << 21, 1 << 14, 1 << 14, fake, fake, fake, 0, fake, 1 << 16, None)
    assert st == nv.ERR_UNSUPPORTED
    assert L.nvfp4_quantize_noalloc(fake, 1 << 21, 1 << 14, 1 << 14, fake, fake, fake, 0, None) == nv.ERR_UNSUPPORTED
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 1, (1 << 23) + 1, 1, 128)  # (2^23 + 1) * 128 > 2^30
    assert L.nvfp4_kv_append(ctypes.byref(kv), 0, fake, fake, fake, 1 << 30, None) == nv.ERR_UNSUPPORTED
    # attention: the key tiles of the whole list are counted in 32 bits
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 1, 1 << 18, 1, 128)  # 2048 tiles per slot
    st = L.nvfp4_kv_attention(ctypes.byref(kv), fake, 1 << 20, fake, 128, ctypes.c_float(0.0), fake, fake, 256, None)
    assert st == nv.ERR_UNSUPPORTED
    # and its work units (pairs of 128-query tiles x heads): 2^12 pairs x 2^20 heads = 2^32
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 1, 128, 1 << 20, 128)
    st = L.nvfp4_kv_attention(ctypes.byref(kv), fake, 1, fake, 1 << 20, ctypes.c_float(0.0), fake, fake, 256, None)
    assert st == nv.ERR_UNSUPPORTED
    # the keys' RoPE tables: present, 16-byte aligned, and 32-bit flat indexes
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 8, 2, 32)
    rope = L.nvfp4_kv_append_rope
    assert rope(ctypes.byref(kv), 0, fake, fake, None, fake, fake, 1 << 16, None) == nv.ERR_INVALID_ARG
    assert rope(ctypes.byref(kv), 0, fake, fake, fake + 4, fake, fake, 1 << 16, None) == nv.ERR_MISALIGNED
    kv = nv.CKVCache(fake, fake, fake, fake, fake, fake, 4, 1 << 20, 16, 128)
    assert rope(ctypes.byref(kv), 0, fake, fake, fake, fake, fake, 1 << 30, None) == nv.ERR_UNSUPPORTED
    # training-side operands: shapes, outputs, signs and alignment are checked before any launch
    q2 = L.nvfp4_quantize_2d
    assert q2(fake, 96, 64, 64, fake, fake, fake, fake, fake, 0, fake, 256, None) == nv.ERR_UNSUPPORTED  # rows % 64
    assert q2(fake, 64, 48, 48, fake, fake, fake, fake, fake, 0, fake, 256, None) == nv.ERR_UNSUPPORTED  # cols % 64
    assert q2(fake, 64, 64, 64, None, None, None, None, fake, 0, fake, 256, None) == nv.ERR_INVALID_ARG  # no output
    assert q2(fake, 64, 64, 64, fake, None, None, None, fake, 0, fake, 256, None) == nv.ERR_INVALID_ARG  # half a pair
    assert q2(fake, 64, 64, 64, fake + 8, fake, None, None, fake, 0, fake, 256, None) == nv.ERR_MISALIGNED
    assert q2(fake, 64, 64, 64, fake, fake, None, None, fake, 0, fake, 16, None) == nv.ERR_INVALID_ARG  # workspace
    qt = L.nvfp4_quantize_t
    assert qt(fake, 64, 24, 24, fake, fake, fake, None, 0, fake, 256, None) == nv.ERR_UNSUPPORTED  # cols % 16
    bad = (ctypes.c_int8 * 16)(*([1] * 15 + [2]))
    assert qt(fake, 64, 32, 32, fake, fake, fake, bad, 0, fake, 256, None) == nv.ERR_INVALID_ARG  # sign not +-1
    assert qt(fake, 64, 32, 32, fake, fake, fake, None, 2, fake, 256, None) == nv.ERR_INVALID_ARG  # unknown flag
    assert qt(fake, 64, 32, 36, fake, fake, fake, None, 0, fake, 256, None) == nv.ERR_MISALIGNED  # ld % 8


def test_product_path_does_not_import_the_oracle():
    pkg = os.path.join(ROOT, "bit_video_dit_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                src = open(os.path.join(dirpath, f), encoding="utf-8").read()
                assert not re.search(r"^\s*(import|from)\s+oracle\b", src, re.M), f
                assert "nvfp4_oracle" not in src and "liboracle" not in src, f
