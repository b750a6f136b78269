"""The W4A4 linear stack of a DiT: L layers of QKV, out-projection, FFN up and
FFN down linears, every hop between them an NVFP4 tensor written by the
previous GEMM's epilogue.

Source: "LongLive-2.0：用 NVFP4 并行底座做长视频生成" (yingwang.github.io reading
note), sections "NVFP4 训练的工程细节" and "推理底座": the model's linears run as
W4A4 NVFP4 GEMMs through self-written kernels, weights and activations both
4-bit; the anzhuoshouzhuan.com LongLive 2.0 article, section "NVFP4 量化", on
fusing the surrounding element-wise work into the kernels.

Per layer (hidden D, FFN width F, M tokens), on the library's calls only:
  qkv  = nvfp4_gemm(x, W_qkv) + b_qkv    -> bf16 [M, 3D] (Q, K, V for the
         attention and the KV append), and its V third (columns 2D .. 3D-1)
         requantized in the same epilogue as the stand-in for the attention
         output (attention, norms and residuals are outside this stack)
  h    = nvfp4_gemm(v, W_out) + b_out    -> NVFP4 [M, D]
  u    = GELU(nvfp4_gemm(h, W_up) + b_up) -> NVFP4 [M, F]
  x'   = nvfp4_gemm(u, W_down) + b_down  -> NVFP4 [M, D], the next layer's input
Each requant uses a fixed output tensor scale (delayed scaling): calibrate()
measures max |y| of every GEMM's output once (out_amax) and sets
a32_out = amax / 2688.  This module only sequences library calls; it holds no
arithmetic of its own.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import nvfp4 as nv

QKV, OUT, UP, DOWN = range(4)


@dataclass
class Layer:
    w: list  # NVFP4Tensor per GEMM (QKV, OUT, UP, DOWN)
    b: list  # bf16 [N] bias per GEMM


class LinearStack:
    """Holds the NVFP4 weights, the output tensor scales and the activation
    buffers of an L-layer stack for M tokens, and runs it on a stream."""

    def __init__(self, M: int, D: int, F: int, device="cuda", qkv_bf16: bool = True):
        self.M, self.D, self.F = M, D, F
        self.device = torch.device(device)
        self.layers: list[Layer] = []
        self.qkv_bf16 = qkv_bf16
        dev = self.device
        self.x_in = nv.empty_nvfp4(M, D, dev)   # the first layer's input (tensor scale computed)
        self.x = nv.empty_nvfp4(M, D, dev)      # each later layer's input; the last layer's output
        self.v = nv.empty_nvfp4(M, D, dev)      # V third of the QKV output
        self.h = nv.empty_nvfp4(M, D, dev)      # out-projection output
        self.u = nv.empty_nvfp4(M, F, dev)      # FFN hidden
        self.qkv = torch.empty((M, 3 * D), dtype=torch.bfloat16, device=dev) if qkv_bf16 else None
        self.ws_q = nv.workspace(nv.OP_QUANTIZE, M, 0, D, dev)
        self.ws_g = nv.workspace(nv.OP_GEMM, M, F, F, dev)
        self.alpha = None  # [L, 4] binary32 output tensor scales (set by calibrate)

    def add_layer(self, weights_bf16: dict, biases_bf16: dict, stream=None) -> None:
        """Quantize one layer's bf16 weights on the device (each with its own
        tensor scale) and keep them with the bf16 biases.  weights_bf16 /
        biases_bf16: device tensors keyed 'qkv', 'out', 'up', 'down'."""
        names = ("qkv", "out", "up", "down")
        w = [nv.quantize(weights_bf16[n], stream=stream) for n in names]
        b = [biases_bf16[n].contiguous() for n in names]
        self.layers.append(Layer(w, b))

    # -- one GEMM of the stack -------------------------------------------
    def _out_of(self, g: int):
        return {QKV: self.v, OUT: self.h, UP: self.u, DOWN: self.x}[g]

    def _in_of(self, l: int, g: int):
        return {QKV: self.x_in if l == 0 else self.x, OUT: self.v, UP: self.h, DOWN: self.u}[g]

    def gemm(self, l: int, g: int, *, requant: bool = True, out_amax=None, debug_y=None, stream=None):
        """GEMM g of layer l with its epilogue: bias (and GELU for UP), the
        NVFP4 requant of its output into the next GEMM's input (QKV: its V
        third), bf16 Q, K, V for QKV.  out_amax / debug_y as nvfp4_gemm's."""
        lay = self.layers[l]
        D = self.D
        q = self._out_of(g)
        if requant:
            q.global_scale = self.alpha[l, g:g + 1]
        window = (2 * D, D) if g == QKV else None
        c = self.qkv if g == QKV else None
        return nv.gemm(self._in_of(l, g), lay.w[g], out=c, bf16_out=c is not None, bias=lay.b[g],
                       act=nv.ACT_GELU_TANH if g == UP else nv.ACT_NONE, requant=q if requant else None,
                       out_amax=out_amax, debug_y=debug_y, out_window=window, ws=self.ws_g, stream=stream)

    def quantize_input(self, x_bf16: torch.Tensor, stream=None) -> None:
        """The first layer's input: bf16 [M, D] -> NVFP4 (tensor scale computed)."""
        nv.quantize(x_bf16, out=self.x_in, ws=self.ws_q, stream=stream)

    def calibrate(self, x_bf16: torch.Tensor) -> None:
        """One pass that fixes every GEMM's output tensor scale: run the GEMM
        with out_amax (over the requantized columns), set a32_out = amax / 2688
        (the same rule as a computed tensor scale), then run it with the
        requant so the next GEMM sees its real input."""
        L = len(self.layers)
        self.alpha = torch.zeros((L, 4), dtype=torch.float32, device=self.device)
        amax = torch.zeros((L, 4), dtype=torch.float32, device=self.device)
        self.quantize_input(x_bf16)
        keep = self.qkv
        if self.qkv is None:
            self.qkv = torch.empty((self.M, 3 * self.D), dtype=torch.bfloat16, device=self.device)
        for l in range(L):
            for g in range(4):
                if g != QKV:
                    # a bf16 output only to run the epilogue (its amax is what is wanted)
                    tmp = torch.empty((self.M, self.layers[l].w[g].rows), dtype=torch.bfloat16, device=self.device)
                    nv.gemm(self._in_of(l, g), self.layers[l].w[g], out=tmp, bias=self.layers[l].b[g],
                            act=nv.ACT_GELU_TANH if g == UP else nv.ACT_NONE, out_amax=amax[l, g:g + 1],
                            ws=self.ws_g)
                    del tmp
                else:
                    nv.gemm(self._in_of(l, g), self.layers[l].w[g], out=self.qkv, bias=self.layers[l].b[g],
                            out_amax=amax[l, g:g + 1], out_window=(2 * self.D, self.D), ws=self.ws_g)
                torch.div(amax[l, g:g + 1], 2688.0, out=self.alpha[l, g:g + 1])
                self.gemm(l, g)
        self.qkv = keep

    def forward(self, x_bf16: torch.Tensor | None = None, stream=None) -> nv.NVFP4Tensor:
        """Quantize x (when given; else self.x_in already holds the input) and
        run every layer; the result is the last layer's NVFP4 output (self.x)."""
        if self.alpha is None:
            raise RuntimeError("calibrate() first: the requants need their output tensor scales")
        if x_bf16 is not None:
            self.quantize_input(x_bf16, stream=stream)
        for l in range(len(self.layers)):
            for g in range(4):
                self.gemm(l, g, stream=stream)
        return self.x

    def flops(self) -> float:
        """2 M N K summed over every GEMM of the stack."""
        M, D, F = self.M, self.D, self.F
        return len(self.layers) * 2.0 * M * (3 * D * D + D * D + F * D + D * F)

    def launches_per_forward(self, with_input: bool = True) -> int:
        return 4 * len(self.layers) + (1 if with_input else 0)
