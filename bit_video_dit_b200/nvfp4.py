"""Thin Python binding of libnvfp4.so (the C ABI declared in include/nvfp4.h).

Argument marshalling only: PyTorch supplies device memory and the current CUDA
stream; every step of quantize / GEMM / KV append / KV dequant runs in the
library's CUDA kernels.  There is no CPU fallback: if the library cannot be
loaded, or no CUDA device is present, the calls raise.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libnvfp4.so")

OK, ERR_INVALID_ARG, ERR_UNSUPPORTED, ERR_MISALIGNED, ERR_CUDA, ERR_TIMEOUT, ERR_DEVICE = range(7)
(OP_QUANTIZE, OP_GEMM, OP_KV_APPEND, OP_KV_DEQUANT, OP_LN_QUANTIZE, OP_QUANTIZE_2D, OP_QUANTIZE_T,
 OP_KV_ATTENTION) = range(8)
Q_COMPUTE_GLOBAL, Q_GIVEN_GLOBAL, Q_ROWMAJOR_SCALES, Q_SCALE_SEARCH = 0, 1, 2, 4
KV_SCALE_SEARCH, KV_SMOOTH_K, KV_SMOOTH_V = 1, 2, 4
ACT_NONE, ACT_GELU_TANH = 0, 1
DBG_SKIP_LOADS = 1

EXPORTS = ("nvfp4_status_string", "nvfp4_version", "nvfp4_codes_bytes", "nvfp4_scales_bytes",
           "nvfp4_workspace_bytes", "nvfp4_read_device_error", "nvfp4_quantize", "nvfp4_gemm",
           "nvfp4_kv_append", "nvfp4_kv_dequant", "nvfp4_test_encode", "nvfp4_quantize_noalloc",
           "nvfp4_ln_modulate_quantize", "nvfp4_quantize_2d", "nvfp4_quantize_t", "nvfp4_attention_chunks",
           "nvfp4_kv_attention", "nvfp4_kv_append_rope")


class NVFP4Error(RuntimeError):
    def __init__(self, fn: str, status: int, msg: str):
        super().__init__(f"{fn} failed: status {status} ({msg})")
        self.status = status


class CTensor(ctypes.Structure):
    _fields_ = [("codes", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("global_scale", ctypes.c_void_p),
                ("rows", ctypes.c_int64), ("cols", ctypes.c_int64)]


class CEpilogue(ctypes.Structure):
    _fields_ = [("bias", ctypes.c_void_p), ("mod_scale", ctypes.c_void_p), ("mod_shift", ctypes.c_void_p),
                ("gate", ctypes.c_void_p), ("residual", ctypes.c_void_p), ("ld_residual", ctypes.c_int64),
                ("act", ctypes.c_int), ("out_codes", ctypes.c_void_p), ("out_scales", ctypes.c_void_p),
                ("out_global_scale", ctypes.c_void_p), ("out_amax", ctypes.c_void_p),
                ("debug_y", ctypes.c_void_p), ("debug_flags", ctypes.c_uint), ("wait_limit_us", ctypes.c_uint32),
                ("out_col0", ctypes.c_int64), ("out_cols", ctypes.c_int64)]


class CKVCache(ctypes.Structure):
    _fields_ = [("k_codes", ctypes.c_void_p), ("k_scales", ctypes.c_void_p), ("v_codes", ctypes.c_void_p),
                ("v_scales", ctypes.c_void_p), ("k_global", ctypes.c_void_p), ("v_global", ctypes.c_void_p),
                ("n_slots", ctypes.c_int32), ("tokens_per_slot", ctypes.c_int32), ("heads", ctypes.c_int32),
                ("head_dim", ctypes.c_int32), ("flags", ctypes.c_uint32), ("k_mean", ctypes.c_void_p),
                ("v_mean", ctypes.c_void_p)]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libnvfp4.so (raises if it has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libnvfp4.so is not built ({LIB_PATH}); run python -m bit_video_dit_b200.build")
        L = ctypes.CDLL(LIB_PATH)
        vp, i64, i32, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32, ctypes.c_size_t
        st = ctypes.c_int
        L.nvfp4_status_string.argtypes = [st]
        L.nvfp4_status_string.restype = ctypes.c_char_p
        L.nvfp4_version.restype = ctypes.c_int
        L.nvfp4_codes_bytes.argtypes = [i64, i64]
        L.nvfp4_codes_bytes.restype = sz
        L.nvfp4_scales_bytes.argtypes = [i64, i64, ctypes.c_int]
        L.nvfp4_scales_bytes.restype = sz
        L.nvfp4_workspace_bytes.argtypes = [ctypes.c_int, i64, i64, i64]
        L.nvfp4_workspace_bytes.restype = sz
        L.nvfp4_read_device_error.argtypes = [vp, vp, ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_uint32)]
        L.nvfp4_read_device_error.restype = st
        L.nvfp4_quantize.argtypes = [vp, i64, i64, i64, vp, vp, vp, ctypes.c_uint, vp, sz, vp]
        L.nvfp4_quantize.restype = st
        L.nvfp4_gemm.argtypes = [ctypes.POINTER(CTensor), ctypes.POINTER(CTensor), vp, i64,
                                 ctypes.POINTER(CEpilogue), vp, sz, vp]
        L.nvfp4_gemm.restype = st
        L.nvfp4_kv_append.argtypes = [ctypes.POINTER(CKVCache), i32, vp, vp, vp, sz, vp]
        L.nvfp4_kv_append.restype = st
        L.nvfp4_kv_append_rope.argtypes = [ctypes.POINTER(CKVCache), i32, vp, vp, vp, vp, vp, sz, vp]
        L.nvfp4_kv_append_rope.restype = st
        L.nvfp4_kv_dequant.argtypes = [ctypes.POINTER(CKVCache), vp, i32, vp, vp, vp, sz, vp]
        L.nvfp4_kv_dequant.restype = st
        L.nvfp4_test_encode.argtypes = [vp, i64, vp, vp, vp]
        L.nvfp4_test_encode.restype = st
        L.nvfp4_quantize_noalloc.argtypes = [vp, i64, i64, i64, vp, vp, vp, ctypes.c_uint, vp]
        L.nvfp4_quantize_noalloc.restype = st
        L.nvfp4_ln_modulate_quantize.argtypes = [vp, i64, i64, i64, vp, vp, ctypes.c_float, vp, vp, vp,
                                                 ctypes.c_uint, vp, sz, vp]
        L.nvfp4_ln_modulate_quantize.restype = st
        L.nvfp4_quantize_2d.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, vp, ctypes.c_uint, vp, sz, vp]
        L.nvfp4_quantize_2d.restype = st
        L.nvfp4_quantize_t.argtypes = [vp, i64, i64, i64, vp, vp, vp, vp, ctypes.c_uint, vp, sz, vp]
        L.nvfp4_quantize_t.restype = st
        L.nvfp4_attention_chunks.argtypes = [i32, i32, i32, i32, i32, ctypes.POINTER(ctypes.c_int32), i32]
        L.nvfp4_attention_chunks.restype = i32
        L.nvfp4_kv_attention.argtypes = [ctypes.POINTER(CKVCache), vp, i32, vp, i32, ctypes.c_float, vp, vp, sz, vp]
        L.nvfp4_kv_attention.restype = st
        _lib = L
    return _lib


def status_string(s: int) -> str:
    return lib().nvfp4_status_string(int(s)).decode()


def _check(fn: str, s: int) -> None:
    if s != OK:
        raise NVFP4Error(fn, s, status_string(s))


def _stream(stream=None) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t: torch.Tensor | None):
    return None if t is None else t.data_ptr()


def _require_cuda(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise ValueError("libnvfp4 works on CUDA tensors only")


def codes_bytes(rows: int, cols: int) -> int:
    return int(lib().nvfp4_codes_bytes(rows, cols))


def scales_bytes(rows: int, cols: int, swizzled: bool = True) -> int:
    return int(lib().nvfp4_scales_bytes(rows, cols, 1 if swizzled else 0))


def workspace_bytes(op: int, m: int = 0, n: int = 0, k: int = 0) -> int:
    return int(lib().nvfp4_workspace_bytes(op, m, n, k))


def workspace(op: int, m: int = 0, n: int = 0, k: int = 0, device="cuda") -> torch.Tensor:
    # zeroed: the first 16 bytes are the device error record
    return torch.zeros(workspace_bytes(op, m, n, k), dtype=torch.uint8, device=device)


def read_device_error(ws: torch.Tensor, stream=None) -> tuple[int, int]:
    code = ctypes.c_int(0)
    info = ctypes.c_uint32(0)
    _check("nvfp4_read_device_error",
           lib().nvfp4_read_device_error(ws.data_ptr(), _stream(stream), ctypes.byref(code), ctypes.byref(info)))
    return code.value, info.value


@dataclass
class NVFP4Tensor:
    """An NVFP4 tensor on the device: packed E2M1 codes [rows, cols/2] (uint8),
    block scales (uint8, swizzled GEMM layout unless rowmajor) and the binary32
    tensor scale (1-element float32 tensor)."""
    codes: torch.Tensor
    scales: torch.Tensor
    global_scale: torch.Tensor
    rows: int
    cols: int

    def c(self) -> CTensor:
        return CTensor(self.codes.data_ptr(), self.scales.data_ptr(), self.global_scale.data_ptr(),
                       self.rows, self.cols)


def empty_nvfp4(rows: int, cols: int, device="cuda", swizzled: bool = True) -> NVFP4Tensor:
    return NVFP4Tensor(torch.empty((rows, cols // 2), dtype=torch.uint8, device=device),
                       torch.empty(scales_bytes(rows, cols, swizzled), dtype=torch.uint8, device=device),
                       torch.empty(1, dtype=torch.float32, device=device), rows, cols)


def quantize(x: torch.Tensor, *, global_scale: torch.Tensor | None = None, out: NVFP4Tensor | None = None,
             rowmajor_scales: bool = False, scale_search: bool = False, ws: torch.Tensor | None = None,
             stream=None) -> NVFP4Tensor:
    """bf16 [rows, cols] (row stride x.stride(0)) -> NVFP4Tensor.  With
    global_scale given, that tensor scale is used (delayed scaling); otherwise
    it is computed as amax / 2688 and written to out.global_scale."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("quantize takes a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    if out is None:
        out = empty_nvfp4(rows, cols, x.device, swizzled=not rowmajor_scales)
    flags = (Q_ROWMAJOR_SCALES if rowmajor_scales else 0) | (Q_SCALE_SEARCH if scale_search else 0)
    if global_scale is not None:
        out.global_scale.copy_(global_scale.reshape(1))
        flags |= Q_GIVEN_GLOBAL
    if ws is None:
        ws = workspace(OP_QUANTIZE, rows, 0, cols, x.device)
    _check("nvfp4_quantize", lib().nvfp4_quantize(
        x.data_ptr(), rows, cols, x.stride(0), out.codes.data_ptr(), out.scales.data_ptr(),
        out.global_scale.data_ptr(), flags, ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def quantize_2d(x: torch.Tensor, *, global_scale: torch.Tensor | None = None, want_rows: bool = True,
                want_t: bool = True, out: NVFP4Tensor | None = None, out_t: NVFP4Tensor | None = None,
                ws: torch.Tensor | None = None, stream=None):
    """2D (16 x 16 block) scaling of a bf16 weight [rows, cols]: returns
    (operand of x, operand of x^T), either None when not wanted; both share the
    tensor scale (computed as amax / 2688 unless global_scale is given)."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("quantize_2d takes a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    a = (out or empty_nvfp4(rows, cols, x.device)) if want_rows else None
    t = (out_t or empty_nvfp4(cols, rows, x.device)) if want_t else None
    gs = (a or t).global_scale
    flags = 0
    if global_scale is not None:
        gs.copy_(global_scale.reshape(1))
        flags |= Q_GIVEN_GLOBAL
    if ws is None:
        ws = workspace(OP_QUANTIZE_2D, rows, 0, cols, x.device)
    _check("nvfp4_quantize_2d", lib().nvfp4_quantize_2d(
        x.data_ptr(), rows, cols, x.stride(0), _ptr(a.codes if a else None), _ptr(a.scales if a else None),
        _ptr(t.codes if t else None), _ptr(t.scales if t else None), gs.data_ptr(), flags, ws.data_ptr(),
        ws.numel(), _stream(stream)))
    if a is not None and t is not None:
        t.global_scale = a.global_scale
    return a, t


def quantize_t(x: torch.Tensor, *, rht_sign=None, global_scale: torch.Tensor | None = None,
               out: NVFP4Tensor | None = None, ws: torch.Tensor | None = None, stream=None) -> NVFP4Tensor:
    """The operand of a GEMM contracting over x's rows (bf16 [rows, cols]):
    x^T quantized with 1D blocks along the rows, after the 16-point Random
    Hadamard Transform when rht_sign (16 values of +1 / -1) is given."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("quantize_t takes a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    if out is None:
        out = empty_nvfp4(cols, rows, x.device)
    flags = 0
    if global_scale is not None:
        out.global_scale.copy_(global_scale.reshape(1))
        flags |= Q_GIVEN_GLOBAL
    if ws is None:
        ws = workspace(OP_QUANTIZE_T, rows, 0, cols, x.device)
    sign = None
    if rht_sign is not None:
        sign = (ctypes.c_int8 * 16)(*[int(v) for v in rht_sign])
    _check("nvfp4_quantize_t", lib().nvfp4_quantize_t(
        x.data_ptr(), rows, cols, x.stride(0), out.codes.data_ptr(), out.scales.data_ptr(),
        out.global_scale.data_ptr(), sign, flags, ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def ln_modulate_quantize(x: torch.Tensor, *, mod_scale: torch.Tensor | None = None,
                         mod_shift: torch.Tensor | None = None, eps: float = 1e-6,
                         global_scale: torch.Tensor | None = None, out: NVFP4Tensor | None = None,
                         rowmajor_scales: bool = False, scale_search: bool = False, ws: torch.Tensor | None = None,
                         stream=None) -> NVFP4Tensor:
    """LayerNorm (no affine) of each row of bf16 x [rows, cols], then
    h * (1 + mod_scale) + mod_shift (bf16 [cols] each, optional), quantized to
    NVFP4 in the same pass (tensor scale from max |m| unless global_scale is given)."""
    _require_cuda(x)
    if x.dtype != torch.bfloat16 or x.dim() != 2 or x.stride(1) != 1:
        raise ValueError("ln_modulate_quantize takes a 2-D bf16 tensor with unit column stride")
    rows, cols = x.shape
    for v in (mod_scale, mod_shift):
        if v is not None and (v.dtype != torch.bfloat16 or v.numel() != cols or not v.is_contiguous()):
            raise ValueError("mod_scale / mod_shift are contiguous bf16 [cols]")
    if out is None:
        out = empty_nvfp4(rows, cols, x.device, swizzled=not rowmajor_scales)
    flags = (Q_ROWMAJOR_SCALES if rowmajor_scales else 0) | (Q_SCALE_SEARCH if scale_search else 0)
    if global_scale is not None:
        out.global_scale.copy_(global_scale.reshape(1))
        flags |= Q_GIVEN_GLOBAL
    if ws is None:
        ws = workspace(OP_LN_QUANTIZE, rows, 0, cols, x.device)
    _check("nvfp4_ln_modulate_quantize", lib().nvfp4_ln_modulate_quantize(
        x.data_ptr(), rows, cols, x.stride(0), _ptr(mod_scale), _ptr(mod_shift), float(eps), out.codes.data_ptr(),
        out.scales.data_ptr(), out.global_scale.data_ptr(), flags, ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


def make_epilogue(*, bias=None, mod_scale=None, mod_shift=None, gate=None, residual=None, act: int = ACT_NONE,
                  requant: NVFP4Tensor | None = None, out_amax=None, debug_y=None, debug_flags: int = 0,
                  wait_limit_us: int = 0, out_window: tuple[int, int] | None = None) -> CEpilogue:
    col0, cols = out_window if out_window is not None else (0, 0)
    return CEpilogue(_ptr(bias), _ptr(mod_scale), _ptr(mod_shift), _ptr(gate), _ptr(residual),
                     0 if residual is None else residual.stride(0), int(act),
                     None if requant is None else requant.codes.data_ptr(),
                     None if requant is None else requant.scales.data_ptr(),
                     None if requant is None else requant.global_scale.data_ptr(),
                     _ptr(out_amax), _ptr(debug_y), int(debug_flags), int(wait_limit_us), int(col0), int(cols))


def gemm(a: NVFP4Tensor, b: NVFP4Tensor, *, out: torch.Tensor | None = None, bias=None, mod_scale=None,
         mod_shift=None, gate=None, residual=None, act: int = ACT_NONE, requant: NVFP4Tensor | None = None,
         out_amax=None, debug_y=None, debug_flags: int = 0, wait_limit_us: int = 0, bf16_out: bool = True,
         out_window: tuple[int, int] | None = None, ws: torch.Tensor | None = None,
         stream=None) -> torch.Tensor | None:
    """C[M, N] = a32_A a32_B (A . S_A)(B . S_B)^T -> epilogue -> bf16 `out`
    and/or NVFP4 `requant` (whose global_scale holds the output tensor scale).
    out_window = (col0, cols): the requant and out_amax cover columns
    col0 .. col0 + cols - 1 only (requant is then an [M, cols] operand)."""
    M, N = a.rows, b.rows
    dev = a.codes.device
    if out is None and bf16_out:
        out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ep = make_epilogue(bias=bias, mod_scale=mod_scale, mod_shift=mod_shift, gate=gate, residual=residual, act=act,
                       requant=requant, out_amax=out_amax, debug_y=debug_y, debug_flags=debug_flags,
                       wait_limit_us=wait_limit_us, out_window=out_window)
    if ws is None:
        ws = workspace(OP_GEMM, M, N, a.cols, dev)
    ca, cb = a.c(), b.c()
    _check("nvfp4_gemm", lib().nvfp4_gemm(ctypes.byref(ca), ctypes.byref(cb), _ptr(out),
                                          0 if out is None else out.stride(0), ctypes.byref(ep),
                                          ws.data_ptr(), ws.numel(), _stream(stream)))
    return out


class KVCache:
    """Paged NVFP4 KV cache: n_slots frame-chunks of tokens x heads x head_dim,
    K and V each stored as codes + row-major E4M3 scales + one binary32 tensor
    scale per slot (9/16 byte per element per tensor).  smooth_k / smooth_v
    add K-smoothing: one binary32 mean per channel (heads x head_dim) per slot."""

    def __init__(self, n_slots: int, tokens: int, heads: int, head_dim: int, device="cuda",
                 scale_search: bool = False, smooth_k: bool = False, smooth_v: bool = False):
        self.n_slots, self.tokens, self.heads, self.head_dim = n_slots, tokens, heads, head_dim
        self.flags = ((KV_SCALE_SEARCH if scale_search else 0) | (KV_SMOOTH_K if smooth_k else 0) |
                      (KV_SMOOTH_V if smooth_v else 0))
        e = tokens * heads * head_dim
        self.slot_elems = e
        u8 = torch.uint8
        self.k_codes = torch.zeros((n_slots, e // 2), dtype=u8, device=device)
        self.v_codes = torch.zeros((n_slots, e // 2), dtype=u8, device=device)
        self.k_scales = torch.zeros((n_slots, e // 16), dtype=u8, device=device)
        self.v_scales = torch.zeros((n_slots, e // 16), dtype=u8, device=device)
        self.k_global = torch.zeros(n_slots, dtype=torch.float32, device=device)
        self.v_global = torch.zeros(n_slots, dtype=torch.float32, device=device)
        f32 = torch.float32
        self.k_mean = torch.zeros((n_slots, heads * head_dim), dtype=f32, device=device) if smooth_k else None
        self.v_mean = torch.zeros((n_slots, heads * head_dim), dtype=f32, device=device) if smooth_v else None
        self.ws_append = workspace(OP_KV_APPEND, tokens * heads, 0, head_dim, device)
        self.ws_dequant = workspace(OP_KV_DEQUANT, device=device)

    def c(self) -> CKVCache:
        return CKVCache(self.k_codes.data_ptr(), self.k_scales.data_ptr(), self.v_codes.data_ptr(),
                        self.v_scales.data_ptr(), self.k_global.data_ptr(), self.v_global.data_ptr(),
                        self.n_slots, self.tokens, self.heads, self.head_dim, self.flags,
                        None if self.k_mean is None else self.k_mean.data_ptr(),
                        None if self.v_mean is None else self.v_mean.data_ptr())

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in
                   (self.k_codes, self.v_codes, self.k_scales, self.v_scales, self.k_global, self.v_global,
                    self.k_mean, self.v_mean) if t is not None)

    def append(self, slot: int, k: torch.Tensor, v: torch.Tensor, stream=None, rope=None) -> None:
        """Quantize one chunk's K and V (bf16 [T, H, d], contiguous) into `slot` in place.
        rope = (cos, sin), device float32 [T, d/2] each: the keys' rotary embedding
        (interleaved pairs) is applied ahead of their quantize (nvfp4_kv_append_rope)."""
        _require_cuda(k, v)
        for t in (k, v):
            if t.dtype != torch.bfloat16 or not t.is_contiguous() or t.numel() != self.slot_elems:
                raise ValueError("append takes contiguous bf16 [T, H, d] chunks")
        cc = self.c()
        if rope is None:
            _check("nvfp4_kv_append", lib().nvfp4_kv_append(
                ctypes.byref(cc), int(slot), k.data_ptr(), v.data_ptr(), self.ws_append.data_ptr(),
                self.ws_append.numel(), _stream(stream)))
            return
        cos, sin = rope
        _require_cuda(cos, sin)
        for t in (cos, sin):
            if t.dtype != torch.float32 or not t.is_contiguous() or t.shape != (self.tokens, self.head_dim // 2):
                raise ValueError("rope tables are contiguous float32 [T, d/2]")
        _check("nvfp4_kv_append_rope", lib().nvfp4_kv_append_rope(
            ctypes.byref(cc), int(slot), k.data_ptr(), v.data_ptr(), cos.data_ptr(), sin.data_ptr(),
            self.ws_append.data_ptr(), self.ws_append.numel(), _stream(stream)))

    def dequant(self, slots: torch.Tensor, k_out: torch.Tensor | None = None, v_out: torch.Tensor | None = None,
                stream=None):
        """Gather the slots listed in `slots` (device int32) back to bf16 [n, T, H, d] K and V."""
        _require_cuda(slots)
        n = slots.numel()
        shape = (n, self.tokens, self.heads, self.head_dim)
        dev = self.k_codes.device
        if k_out is None:
            k_out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        if v_out is None:
            v_out = torch.empty(shape, dtype=torch.bfloat16, device=dev)
        cc = self.c()
        _check("nvfp4_kv_dequant", lib().nvfp4_kv_dequant(
            ctypes.byref(cc), slots.data_ptr(), n, k_out.data_ptr(), v_out.data_ptr(),
            self.ws_dequant.data_ptr(), self.ws_dequant.numel(), _stream(stream)))
        return k_out, v_out

    def attention(self, slots: torch.Tensor, q: torch.Tensor, *, scale: float = 0.0, out: torch.Tensor | None = None,
                  ws: torch.Tensor | None = None, stream=None) -> torch.Tensor:
        """softmax(scale Q K^T) V over every key of the listed slots (device int32), K and V read from
        the NVFP4 cache; q and the result are bf16 [Tq, H, d]; scale 0 means 1 / sqrt(d)."""
        _require_cuda(slots, q)
        if q.dtype != torch.bfloat16 or not q.is_contiguous() or q.dim() != 3 or q.shape[1:] != (self.heads,
                                                                                               self.head_dim):
            raise ValueError("attention takes contiguous bf16 q [Tq, heads, head_dim]")
        if out is None:
            out = torch.empty_like(q)
        if ws is None:
            ws = workspace(OP_KV_ATTENTION, device=q.device)
        cc = self.c()
        _check("nvfp4_kv_attention", lib().nvfp4_kv_attention(
            ctypes.byref(cc), slots.data_ptr(), slots.numel(), q.data_ptr(), q.shape[0], float(scale),
            out.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)))
        return out


def attention_chunks(t: int, sink_global: int, shot_start: int, sink_shot: int, window: int) -> list[int]:
    """Chunk indices step t attends to: the global sink, the shot sink and the window, without
    repeats, ascending (computed by the library's host function)."""
    cap = max(1, t)
    buf = (ctypes.c_int32 * cap)()
    n = lib().nvfp4_attention_chunks(t, sink_global, shot_start, sink_shot, window, buf, cap)
    if n < 0:
        raise ValueError("nvfp4_attention_chunks: bad arguments")
    return list(buf[:n])


def test_encode(x: torch.Tensor, e2m1: bool = True, e4m3: bool = True, stream=None):
    """Run the device encoders on binary32 values (test support)."""
    _require_cuda(x)
    x = x.contiguous().view(-1)
    o1 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device) if e2m1 else None
    o2 = torch.empty(x.numel(), dtype=torch.uint8, device=x.device) if e4m3 else None
    _check("nvfp4_test_encode", lib().nvfp4_test_encode(x.data_ptr(), x.numel(), _ptr(o1), _ptr(o2),
                                                         _stream(stream)))
    return o1, o2
