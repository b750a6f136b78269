"""CPU oracle for the NVFP4 W4A4 linear layer and NVFP4 KV-cache store.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
bench's CPU-baseline / reference leg may import this package.  The product
path (``bit_video_dit_b200``) never imports it and shares no code with it.

The arithmetic lives in ``nvfp4_oracle.c`` (plain C, binary32 steps with
``-ffp-contract=off``, binary64 GEMM accumulation); this module only builds
that file with gcc and marshals numpy arrays through ctypes; the attention over
the cache (its chunk set and fp64 softmax attention) is written out in plain
numpy below.  Format source:
"LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io reading note),
section 二 方法 / "NVFP4 量化格式" (E2M1 codes, per-16 E4M3 block scale, FP32
tensor scale, the Dequant equation) and "推理底座" (per-chunk KV quantization).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
# The planted-mistake tests point these at a modified copy of the C source (and
# a library path of their own) in a child process; nothing else sets them.
_SRC = os.environ.get("NVFP4_ORACLE_SRC") or os.path.join(_HERE, "nvfp4_oracle.c")
_LIB_PATH = os.environ.get("NVFP4_ORACLE_LIB") or os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

MODE_COMPUTE = 0
MODE_GIVEN = 1
MODE_SEARCH46 = 4  # OR-ed into the mode: adaptive scale search over {4, 6} (R18)


def build(force: bool = False) -> str:
    """Compile nvfp4_oracle.c into liboracle.so (gcc, OpenMP, no FP contraction)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=gnu11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp",
           "-fPIC", "-shared", "-fvisibility=hidden", _SRC, "-o", tmp, "-lm"]
    subprocess.check_call(cmd)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


class _Epilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("mod_scale", ctypes.c_void_p),
                ("mod_shift", ctypes.c_void_p), ("gate", ctypes.c_void_p),
                ("residual", ctypes.c_void_p), ("ld_res", ctypes.c_int64),
                ("act", ctypes.c_int)]


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            i64, f32, vp, u16 = ctypes.c_int64, ctypes.c_float, ctypes.c_void_p, ctypes.c_uint16
            L.orc_set_threads.argtypes = [ctypes.c_int]
            L.orc_get_threads.restype = ctypes.c_int
            L.orc_bf16_to_f32.argtypes = [u16]
            L.orc_bf16_to_f32.restype = f32
            L.orc_f64_to_bf16.argtypes = [ctypes.c_double]
            L.orc_f64_to_bf16.restype = u16
            L.orc_f32_to_bf16.argtypes = [f32]
            L.orc_f32_to_bf16.restype = u16
            L.orc_e2m1_value.argtypes = [ctypes.c_uint]
            L.orc_e2m1_value.restype = ctypes.c_double
            L.orc_e4m3_value.argtypes = [ctypes.c_uint]
            L.orc_e4m3_value.restype = ctypes.c_double
            L.orc_e2m1_encode.argtypes = [f32]
            L.orc_e2m1_encode.restype = ctypes.c_uint
            L.orc_e4m3_encode.argtypes = [f32]
            L.orc_e4m3_encode.restype = ctypes.c_uint
            for name in ("orc_quantize_f32", "orc_quantize_bf16"):
                fn = getattr(L, name)
                fn.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, vp, vp]
                fn.restype = ctypes.c_int
            L.orc_swizzled_bytes.argtypes = [i64, i64]
            L.orc_swizzled_bytes.restype = i64
            L.orc_swizzle_offset.argtypes = [i64, i64, i64]
            L.orc_swizzle_offset.restype = i64
            L.orc_swizzle_scales.argtypes = [vp, i64, i64, vp]
            L.orc_unswizzle_scales.argtypes = [vp, i64, i64, vp]
            L.orc_dequant_f32.argtypes = [vp, vp, f32, i64, i64, vp]
            L.orc_dequant_bf16.argtypes = [vp, vp, f32, i64, i64, vp]
            L.orc_gemm.argtypes = [vp, vp, f32, vp, vp, f32, i64, i64, i64,
                                   ctypes.POINTER(_Epilogue), vp, i64, vp, vp]
            L.orc_gemm.restype = ctypes.c_int
            L.orc_gemm_exact_bf16.argtypes = [vp, vp, f32, vp, vp, f32, i64, i64, i64, vp]
            L.orc_gemm_exact_bf16.restype = ctypes.c_int
            L.orc_kv_slot_bytes.argtypes = [i64, i64, i64]
            L.orc_kv_slot_bytes.restype = i64
            L.orc_ln_stats.argtypes = [vp, i64, i64, i64, f32, vp]
            L.orc_ln_stats.restype = ctypes.c_int
            L.orc_ln_modulate_given.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp]
            L.orc_ln_modulate_given.restype = ctypes.c_int
            L.orc_ln_modulate.argtypes = [vp, i64, i64, i64, vp, vp, f32, vp]
            L.orc_ln_modulate.restype = ctypes.c_int
            L.orc_ln_modulate_quantize.argtypes = [vp, i64, i64, i64, vp, vp, f32, vp, ctypes.c_int, vp, vp, vp]
            L.orc_ln_modulate_quantize.restype = ctypes.c_int
            for name in ("orc_kv_append", "orc_kv_append_search46"):
                getattr(L, name).argtypes = [vp, i64, i64, i64, i64, vp, vp, vp]
                getattr(L, name).restype = ctypes.c_int
            L.orc_kv_dequant.argtypes = [vp, vp, f32, i64, i64, i64, vp]
            L.orc_channel_mean.argtypes = [vp, i64, i64, vp]
            L.orc_kv_append_smooth.argtypes = [vp, i64, i64, i64, ctypes.c_int, vp, vp, vp, vp, ctypes.c_int]
            L.orc_kv_append_smooth.restype = ctypes.c_int
            L.orc_kv_dequant_smooth.argtypes = [vp, vp, f32, vp, i64, i64, i64, vp]
            for name in ("orc_quantize_2d_f32", "orc_quantize_2d_bf16"):
                getattr(L, name).argtypes = [vp, i64, i64, ctypes.c_int, vp, vp, vp, vp, vp]
                getattr(L, name).restype = ctypes.c_int
            L.orc_rht16_f32.argtypes = [vp, i64, vp, vp]
            L.orc_rope.argtypes = [vp, i64, i64, i64, vp, vp, vp]
            L.orc_channel_mean_f32.argtypes = [vp, i64, i64, vp]
            L.orc_kv_append_rope.argtypes = [vp, i64, i64, i64, vp, vp, ctypes.c_int, vp, vp, vp, vp, ctypes.c_int]
            L.orc_kv_append_rope.restype = ctypes.c_int
            L.orc_quantize_t_bf16.argtypes = [vp, i64, i64, i64, vp, ctypes.c_int, vp, vp, vp]
            L.orc_quantize_t_bf16.restype = ctypes.c_int
            _lib = L
    return _lib


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data


def set_threads(n: int) -> None:
    lib().orc_set_threads(int(n))


def get_threads() -> int:
    return int(lib().orc_get_threads())


# ---- scalar format helpers ---------------------------------------------------

def e2m1_value(code: int) -> float:
    return float(lib().orc_e2m1_value(int(code)))


def e4m3_value(code: int) -> float:
    return float(lib().orc_e4m3_value(int(code)))


def e2m1_encode(y: float) -> int:
    return int(lib().orc_e2m1_encode(float(np.float32(y))))


def e4m3_encode(r: float) -> int:
    return int(lib().orc_e4m3_encode(float(np.float32(r))))


def f64_to_bf16(x: float) -> int:
    return int(lib().orc_f64_to_bf16(float(x)))


def bf16_to_f32(h: int) -> float:
    return float(lib().orc_bf16_to_f32(int(h)))


# ---- array API ---------------------------------------------------------------

def quantize(x: np.ndarray, alpha: float | None = None, search46: bool = False):
    """Quantize a 2-D array (uint16 bf16 bits or float32).

    Returns (codes uint8 [R, C/2], scales uint8 logical [R, C/16], alpha float32).
    alpha=None computes the tensor scale (R1); otherwise it is used as given.
    search46 adds the per-block adaptive scale search over the targets {4, 6} (R18).
    """
    assert x.ndim == 2
    x = np.ascontiguousarray(x)
    R, C = x.shape
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    a = np.zeros(1, np.float32)
    mode = MODE_COMPUTE
    if alpha is not None:
        a[0] = np.float32(alpha)
        mode = MODE_GIVEN
    if search46:
        mode |= MODE_SEARCH46
    if x.dtype == np.uint16:
        fn = lib().orc_quantize_bf16
    elif x.dtype == np.float32:
        fn = lib().orc_quantize_f32
    else:
        raise TypeError("oracle.quantize takes bf16 bits (uint16) or float32")
    rc = fn(_p(x), R, C, C, mode, _p(a), _p(codes), _p(scales))
    if rc != 0:
        raise ValueError(f"orc_quantize failed ({rc})")
    return codes, scales, np.float32(a[0])


def swizzled_bytes(rows: int, sc: int) -> int:
    return int(lib().orc_swizzled_bytes(rows, sc))


def swizzle_offset(r: int, c: int, sc: int) -> int:
    return int(lib().orc_swizzle_offset(r, c, sc))


def swizzle(scales: np.ndarray) -> np.ndarray:
    scales = np.ascontiguousarray(scales, dtype=np.uint8)
    R, S = scales.shape
    out = np.zeros(swizzled_bytes(R, S), np.uint8)
    lib().orc_swizzle_scales(_p(scales), R, S, _p(out))
    return out


def unswizzle(swz: np.ndarray, rows: int, sc: int) -> np.ndarray:
    swz = np.ascontiguousarray(swz, dtype=np.uint8).reshape(-1)
    assert swz.size >= swizzled_bytes(rows, sc)
    out = np.zeros((rows, sc), np.uint8)
    lib().orc_unswizzle_scales(_p(swz), rows, sc, _p(out))
    return out


def dequant_f32(codes, scales, alpha) -> np.ndarray:
    R = codes.shape[0]
    C = codes.shape[1] * 2
    out = np.zeros((R, C), np.float32)
    lib().orc_dequant_f32(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                          float(alpha), R, C, _p(out))
    return out


def dequant_bf16(codes, scales, alpha) -> np.ndarray:
    R = codes.shape[0]
    C = codes.shape[1] * 2
    out = np.zeros((R, C), np.uint16)
    lib().orc_dequant_bf16(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)),
                           float(alpha), R, C, _p(out))
    return out


def gemm(a, b, *, bias=None, mod_scale=None, mod_shift=None, gate=None, residual=None,
         act: int = 0, rows=None, want_bf16: bool = True):
    """fp64 reference GEMM.  a, b = (codes, logical scales, alpha) triples with
    A [M x K] and B [N x K].  Epilogue vectors are bf16 bits (uint16).
    Returns (y fp64 [R x N], out bf16 bits [R x N] or None)."""
    ac, asc, aa = a
    bc, bsc, ba = b
    M, K = ac.shape[0], ac.shape[1] * 2
    N = bc.shape[0]
    assert bc.shape[1] * 2 == K
    keep = []

    def cp(v):
        if v is None:
            return None
        v = np.ascontiguousarray(v)
        keep.append(v)
        return v.ctypes.data

    ep = _Epilogue(cp(bias), cp(mod_scale), cp(mod_shift), cp(gate), cp(residual),
                   N if residual is None else residual.shape[1], int(act))
    rl = None
    R = M
    if rows is not None:
        rl = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        R = rl.size
    y = np.zeros((R, N), np.float64)
    out = np.zeros((R, N), np.uint16) if want_bf16 else None
    rc = lib().orc_gemm(_p(np.ascontiguousarray(ac)), _p(np.ascontiguousarray(asc)), float(aa),
                        _p(np.ascontiguousarray(bc)), _p(np.ascontiguousarray(bsc)), float(ba),
                        M, N, K, ctypes.byref(ep), _p(rl), R, _p(y), _p(out))
    if rc != 0:
        raise ValueError(f"orc_gemm failed ({rc})")
    return y, out


def gemm_exact_bf16(a, b) -> np.ndarray:
    ac, asc, aa = a
    bc, bsc, ba = b
    M, K = ac.shape[0], ac.shape[1] * 2
    N = bc.shape[0]
    out = np.zeros((M, N), np.uint16)
    rc = lib().orc_gemm_exact_bf16(_p(np.ascontiguousarray(ac)), _p(np.ascontiguousarray(asc)), float(aa),
                                   _p(np.ascontiguousarray(bc)), _p(np.ascontiguousarray(bsc)), float(ba),
                                   M, N, K, _p(out))
    if rc != 0:
        raise ValueError(f"orc_gemm_exact_bf16 failed ({rc})")
    return out


def kv_slot_bytes(T: int, H: int, d: int) -> int:
    return int(lib().orc_kv_slot_bytes(T, H, d))


def kv_append(x: np.ndarray, search46: bool = False):
    """x: bf16 bits [T, H, d].  Returns (codes [T*H, d/2], scales [T*H, d/16], alpha).
    search46 adds the adaptive scale search over the targets {4, 6} (R18)."""
    T, H, d = x.shape
    x = np.ascontiguousarray(x)
    codes = np.zeros((T * H, d // 2), np.uint8)
    scales = np.zeros((T * H, d // 16), np.uint8)
    a = np.zeros(1, np.float32)
    fn = lib().orc_kv_append_search46 if search46 else lib().orc_kv_append
    rc = fn(_p(x), T, H, d, d, _p(codes), _p(scales), _p(a))
    if rc != 0:
        raise ValueError(f"orc_kv_append failed ({rc})")
    return codes, scales, np.float32(a[0])


def kv_dequant(codes, scales, alpha, T: int, H: int, d: int) -> np.ndarray:
    out = np.zeros((T, H, d), np.uint16)
    lib().orc_kv_dequant(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)), float(alpha),
                         T, H, d, _p(out))
    return out


def channel_mean(x: np.ndarray) -> np.ndarray:
    """Binary32 mean over the first axis of bf16 bits x [T, C...] for every
    channel (R20: the binary64 mean rounded once)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    T = x.shape[0]
    C = x.size // T
    mean = np.zeros(C, np.float32)
    lib().orc_channel_mean(_p(x), T, C, _p(mean))
    return mean


def kv_append_smooth(x: np.ndarray, search46: bool = False, mean=None):
    """K-smoothing append (R20): x bf16 bits [T, H, d].  Returns (codes, scales,
    alpha, mean [H*d]); the quantized values are fl32(x - mean[channel]).  With
    `mean` given (binary32 [H*d], e.g. the means a kernel stored) those are
    used instead of the oracle's own."""
    T, H, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    codes = np.zeros((T * H, d // 2), np.uint8)
    scales = np.zeros((T * H, d // 16), np.uint8)
    a = np.zeros(1, np.float32)
    given = mean is not None
    mean = np.array(mean, np.float32).reshape(H * d) if given else np.zeros(H * d, np.float32)
    rc = lib().orc_kv_append_smooth(_p(x), T, H, d, MODE_SEARCH46 if search46 else 0, _p(codes), _p(scales),
                                    _p(a), _p(mean), 1 if given else 0)
    if rc != 0:
        raise ValueError(f"orc_kv_append_smooth failed ({rc})")
    return codes, scales, np.float32(a[0]), mean


def kv_dequant_smooth(codes, scales, alpha, mean, T: int, H: int, d: int) -> np.ndarray:
    """R20 dequant: bf16 of fl32(fl32(fl32(e2m1 * s) * alpha) + mean[channel])."""
    out = np.zeros((T, H, d), np.uint16)
    mean = np.ascontiguousarray(mean, dtype=np.float32)
    lib().orc_kv_dequant_smooth(_p(np.ascontiguousarray(codes)), _p(np.ascontiguousarray(scales)), float(alpha),
                                _p(mean), T, H, d, _p(out))
    return out


def _rope_tables(cos, sin, T: int, d: int):
    cs = np.ascontiguousarray(cos, dtype=np.float32)
    sn = np.ascontiguousarray(sin, dtype=np.float32)
    if cs.shape != (T, d // 2) or sn.shape != (T, d // 2):
        raise ValueError("cos / sin must be [T, d/2]")
    return cs, sn


def rope(x: np.ndarray, cos, sin) -> np.ndarray:
    """R24: bf16 bits x [T, H, d] with every head's interleaved pairs (2p, 2p+1)
    turned by the binary32 angle table (cos, sin [T, d/2]); binary32 [T, H, d]."""
    T, H, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    cs, sn = _rope_tables(cos, sin, T, d)
    y = np.zeros((T, H, d), np.float32)
    lib().orc_rope(_p(x), T, H, d, _p(cs), _p(sn), _p(y))
    return y


def channel_mean_f32(v: np.ndarray) -> np.ndarray:
    """R20's channel mean of binary32 values v [T, C...] (the binary64 mean rounded once)."""
    v = np.ascontiguousarray(v, dtype=np.float32)
    T = v.shape[0]
    C = v.size // T
    mean = np.zeros(C, np.float32)
    lib().orc_channel_mean_f32(_p(v), T, C, _p(mean))
    return mean


def kv_append_rope(x: np.ndarray, cos, sin, smooth: bool = False, search46: bool = False, mean=None):
    """The keys' append with R24 (x bf16 bits [T, H, d]): rope, then (smooth) the
    channel means of the rotated keys taken out (R20; the given binary32 [H*d]
    `mean` instead of the oracle's own when passed), then the quantize.
    Returns (codes, scales, alpha, mean [H*d] or None)."""
    T, H, d = x.shape
    x = np.ascontiguousarray(x, dtype=np.uint16)
    cs, sn = _rope_tables(cos, sin, T, d)
    codes = np.zeros((T * H, d // 2), np.uint8)
    scales = np.zeros((T * H, d // 16), np.uint8)
    a = np.zeros(1, np.float32)
    given = smooth and mean is not None
    if smooth:
        mean = np.array(mean, np.float32).reshape(H * d) if given else np.zeros(H * d, np.float32)
    else:
        mean = None
    rc = lib().orc_kv_append_rope(_p(x), T, H, d, _p(cs), _p(sn), MODE_SEARCH46 if search46 else 0, _p(codes),
                                  _p(scales), _p(a), _p(mean), 1 if given else 0)
    if rc != 0:
        raise ValueError(f"orc_kv_append_rope failed ({rc})")
    return codes, scales, np.float32(a[0]), mean


def quantize_2d(x: np.ndarray, alpha: float | None = None):
    """2D block scaling (R21) of a 2-D array (bf16 bits or float32), rows and cols
    multiples of 16.  Returns (codes [R, C/2], scales [R, C/16], codes_t [C, R/2],
    scales_t [C, R/16], alpha): the row-wise operand and the transposed one."""
    x = np.ascontiguousarray(x)
    R, C = x.shape
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    codes_t = np.zeros((C, R // 2), np.uint8)
    scales_t = np.zeros((C, R // 16), np.uint8)
    a = np.zeros(1, np.float32)
    mode = MODE_COMPUTE
    if alpha is not None:
        a[0] = np.float32(alpha)
        mode = MODE_GIVEN
    fn = {np.dtype(np.uint16): lib().orc_quantize_2d_bf16, np.dtype(np.float32): lib().orc_quantize_2d_f32}[x.dtype]
    rc = fn(_p(x), R, C, mode, _p(a), _p(codes), _p(scales), _p(codes_t), _p(scales_t))
    if rc != 0:
        raise ValueError(f"orc_quantize_2d failed ({rc})")
    return codes, scales, codes_t, scales_t, np.float32(a[0])


def rht16(x: np.ndarray, sign) -> np.ndarray:
    """R22 on each consecutive 16-element block of float32 x (size % 16 == 0)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    sg = np.ascontiguousarray(sign, dtype=np.int8)
    assert sg.size == 16 and x.size % 16 == 0
    out = np.zeros_like(x)
    lib().orc_rht16_f32(_p(x), x.size // 16, _p(sg), _p(out))
    return out


def quantize_t(x: np.ndarray, sign=None, alpha: float | None = None):
    """Transposed operand of bf16 bits x [R, C] (R % 16 == 0): x^T quantized with
    1D blocks along R, after R22 when sign (16 entries of +1/-1) is given.
    Returns (codes_t [C, R/2], scales_t [C, R/16], alpha)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, C = x.shape
    codes = np.zeros((C, R // 2), np.uint8)
    scales = np.zeros((C, R // 16), np.uint8)
    a = np.zeros(1, np.float32)
    mode = MODE_COMPUTE
    if alpha is not None:
        a[0] = np.float32(alpha)
        mode = MODE_GIVEN
    sg = None if sign is None else np.ascontiguousarray(sign, dtype=np.int8)
    rc = lib().orc_quantize_t_bf16(_p(x), R, C, C, None if sg is None else _p(sg), mode, _p(a), _p(codes),
                                   _p(scales))
    if rc != 0:
        raise ValueError(f"orc_quantize_t failed ({rc})")
    return codes, scales, np.float32(a[0])


def attention_chunks(t: int, sink_global: int, shot_start: int, sink_shot: int, window: int) -> list[int]:
    """The chunk indices chunk t attends to in the cache (reading note, section 二, the multi-shot anchors):
    A_g = the video's first sink_global chunks, A_s = the current shot's first sink_shot chunks (the shot starts
    at chunk shot_start), and the window KV[t - window, t); their union without repeats, only chunks already
    made (index < t), ascending."""
    s = set(range(0, sink_global)) | set(range(shot_start, shot_start + sink_shot)) | set(range(t - window, t))
    return sorted(c for c in s if 0 <= c < t)


def _as_f64(x: np.ndarray) -> np.ndarray:
    """bf16 bits (uint16) or binary32 values -> float64."""
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return np.asarray(x, dtype=np.float64)


def attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, scale: float) -> np.ndarray:
    """fp64 softmax attention of q [Tq, H, d] over k, v [L, H, d] (bf16 bits or binary32 values; every query
    sees every key): O[i, h] = sum_j softmax_j(scale * q[i, h] . k[j, h]) v[j, h].  Returns float64 [Tq, H, d]."""
    qf, kf, vf = _as_f64(q), _as_f64(k), _as_f64(v)
    Tq, H, d = qf.shape
    out = np.zeros((Tq, H, d), np.float64)
    for h in range(H):
        s = (qf[:, h, :] @ kf[:, h, :].T) * scale
        s -= s.max(axis=1, keepdims=True)
        p = np.exp(s)
        p /= p.sum(axis=1, keepdims=True)
        out[:, h, :] = p @ vf[:, h, :]
    return out


def ln_stats(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    """R19's row statistics of bf16 bits x [R, C]: binary32 [R, 2] holding
    (mean, rstd) = (fl32(mu), fl32(1 / sqrt(var + eps))), mu and var taken in
    binary64 (population variance)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, C = x.shape
    st = np.zeros((R, 2), np.float32)
    rc = lib().orc_ln_stats(_p(x), R, C, C, float(eps), _p(st))
    if rc != 0:
        raise ValueError(f"orc_ln_stats failed ({rc})")
    return st


def _ln_vecs(scale, shift):
    sc = None if scale is None else np.ascontiguousarray(scale, dtype=np.uint16)
    sh = None if shift is None else np.ascontiguousarray(shift, dtype=np.uint16)
    return sc, sh


def ln_modulate(x: np.ndarray, scale=None, shift=None, eps: float = 1e-6, stats=None) -> np.ndarray:
    """LayerNorm of each row of bf16 bits x [R, C] (no affine), then
    m = h * (1 + scale) + shift (bf16 bits [C] or None), binary32 (R19).  With
    `stats` (binary32 [R, 2] of (mean, rstd), e.g. a kernel's) those row
    statistics are used instead of ln_stats'."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, C = x.shape
    m = np.zeros((R, C), np.float32)
    sc, sh = _ln_vecs(scale, shift)
    if stats is None:
        rc = lib().orc_ln_modulate(_p(x), R, C, C, _p(sc), _p(sh), float(eps), _p(m))
    else:
        st = np.ascontiguousarray(stats, dtype=np.float32).reshape(R, 2)
        rc = lib().orc_ln_modulate_given(_p(x), R, C, C, _p(st), _p(sc), _p(sh), _p(m))
    if rc != 0:
        raise ValueError(f"orc_ln_modulate failed ({rc})")
    return m


def ln_modulate_quantize(x: np.ndarray, scale=None, shift=None, eps: float = 1e-6, alpha: float | None = None,
                         stats=None):
    """ln_modulate then quantize (R19, R1..R8).  Returns (codes, logical scales, alpha)."""
    x = np.ascontiguousarray(x, dtype=np.uint16)
    R, C = x.shape
    codes = np.zeros((R, C // 2), np.uint8)
    scales = np.zeros((R, C // 16), np.uint8)
    a = np.zeros(1, np.float32)
    mode = MODE_COMPUTE
    if alpha is not None:
        a[0] = np.float32(alpha)
        mode = MODE_GIVEN
    sc, sh = _ln_vecs(scale, shift)
    st = None if stats is None else np.ascontiguousarray(stats, dtype=np.float32).reshape(R, 2)
    rc = lib().orc_ln_modulate_quantize(_p(x), R, C, C, _p(sc), _p(sh), float(eps), _p(st), mode, _p(a), _p(codes),
                                        _p(scales))
    if rc != 0:
        raise ValueError(f"orc_ln_modulate_quantize failed ({rc})")
    return codes, scales, np.float32(a[0])
