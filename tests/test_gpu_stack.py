"""The DiT linear stack at full size on the GPU: 30 layers at 16384 tokens,
every hop between GEMMs an NVFP4 tensor written by the previous epilogue:
  QKV 3072->9216 with bias (bf16 Q, K, V; its V third, columns 6144..9215,
  requantized in the same epilogue as the stand-in attention output) ->
  out-proj 3072->3072 + bias, requant -> FFN up 3072->14336 + bias, GELU,
  requant -> FFN down 14336->3072 + bias, requant -> the next layer.
Output tensor scales come from one calibration pass (out_amax over each
requantized window; reading R14).  On sampled rows of every GEMM of every
layer (reading R12, R13):
  * y (the kernel's binary32 result, debug_y) against the oracle's fp64 GEMM
    on the same NVFP4 operands, normwise within 2e-3, and the bf16 output
    (QKV) as bf16(y);
  * every requant bit for bit as the oracle's quantize of those rows of the
    kernel's y with the given output scale;
  * the production check of R13: the requant against the oracle's quantize of
    its own fp64 y: the fraction of codes that differ, each one grid step.
The weights the GPU quantized are checked bit for bit against the oracle's
quantize of the same bf16 weights, and a plain forward (no debug outputs)
reproduces the checked run's final output bit for bit."""
import numpy as np
import pytest
import torch

import oracle
from bit_video_dit_b200 import nvfp4 as nv
from bit_video_dit_b200 import synthetic as syn
from bit_video_dit_b200.stack import QKV, UP, LinearStack

from .gpu_util import GEMM_TOL, dev_bf16, f32_bits, host_bits, host_u8, normwise_err, require_gpu

pytestmark = pytest.mark.gpu

M, L = syn.STACK_M, syn.STACK_LAYERS
D, F = syn.STACK_LAYER[0].K, syn.STACK_LAYER[2].N
ROWS = np.unique(np.concatenate([[0, 1, 127, 128, 255, 256, M - 1], np.random.default_rng(81).integers(0, M, 25)]))
NAMES = ("qkv", "out", "up", "down")

# signed E2M1 grid in code order 0..15 (bit 3 = sign) and each code's rank on the sorted signed grid
E2M1 = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6, -0.0, -0.5, -1, -1.5, -2, -3, -4, -6])
RANK = np.array([7, 8, 9, 10, 11, 12, 13, 14, 7, 6, 5, 4, 3, 2, 1, 0])


def _rows_of(q: nv.NVFP4Tensor, rows_dev):
    """The sampled rows of a device NVFP4 tensor, as oracle operands."""
    codes = host_u8(q.codes.view(q.rows, -1)[rows_dev])
    scales = oracle.unswizzle(host_u8(q.scales), q.rows, q.cols // 16)[ROWS]
    return codes, scales, np.float32(q.global_scale.item())


def _nibbles(codes):
    c = np.asarray(codes, np.uint8)
    return np.stack([c & 0xF, c >> 4], axis=-1).reshape(c.shape[0], -1)


class Mismatch:
    """R13's production comparison: kernel requant vs the oracle's requant of its own y."""

    def __init__(self):
        self.codes = self.code_diff = self.zero_sign = self.blocks = self.scale_diff = 0

    def add(self, got, want):
        gc, gs = _nibbles(got[0]), got[1]
        wc, ws = _nibbles(want[0]), want[1]
        self.blocks += gs.size
        sdiff = gs != ws
        self.scale_diff += int(sdiff.sum())
        # a differing scale is one E4M3 step (adjacent codes of the unsigned scale)
        assert np.all(np.abs(gs[sdiff].astype(int) - ws[sdiff].astype(int)) == 1)
        same = np.repeat(~sdiff, 16, axis=1)
        self.codes += int(same.sum())
        d = (gc != wc) & same
        # +0 against -0 (code 0x0 against 0x8): the same value, counted apart
        z = d & (RANK[gc] == RANK[wc])
        self.zero_sign += int(z.sum())
        d &= ~z
        self.code_diff += int(d.sum())
        # a differing code in a block with the same scale is the neighbouring grid point
        assert np.all(np.abs(RANK[gc[d]] - RANK[wc[d]]) == 1), "a requant code is more than one grid step off"

    def report(self):
        return (f"requant vs the oracle's own requant: {self.code_diff} of {self.codes} codes differ "
                f"({self.code_diff / max(1, self.codes):.2e}), each by one grid step; {self.zero_sign} differ in the "
                f"sign of a zero code only; {self.scale_diff} of {self.blocks} block scales differ "
                f"({self.scale_diff / max(1, self.blocks):.2e}), each by one E4M3 step")


def test_thirty_layer_stack_sampled_rows():
    require_gpu()
    rows_dev = torch.from_numpy(ROWS).cuda()
    x_bits = syn.activations_bf16(M, D, seed=80)
    xd = dev_bf16(x_bits)
    st = LinearStack(M, D, F)
    for l in range(L):
        w, b = syn.stack_layer_bf16(l, D, F)
        st.add_layer({k: dev_bf16(v) for k, v in w.items()}, {k: dev_bf16(v) for k, v in b.items()})
    st.calibrate(xd)
    torch.cuda.synchronize()
    alpha = st.alpha.cpu().numpy()
    assert np.all(alpha > 0)

    # the checked run: the same calls as forward(), each GEMM with debug_y
    st.quantize_input(xd)
    torch.cuda.synchronize()
    oc, osc, oa = oracle.quantize(x_bits)
    assert f32_bits(st.x_in.global_scale.cpu().numpy()) == f32_bits(oa)
    assert np.array_equal(host_u8(st.x_in.codes), oc)
    dy_buf = torch.empty(M * F, dtype=torch.float32, device="cuda")
    mm = Mismatch()
    worst = 0.0
    for l in range(L):
        w, b = syn.stack_layer_bf16(l, D, F)
        ow = []
        for g, n in enumerate(NAMES):
            q = oracle.quantize(w[n])
            wq = st.layers[l].w[g]
            assert f32_bits(wq.global_scale.cpu().numpy()) == f32_bits(q[2]), (l, n)
            assert np.array_equal(host_u8(wq.codes), q[0]), (l, n)
            assert np.array_equal(host_u8(wq.scales), oracle.swizzle(q[1])), (l, n)
            ow.append(q)
        for g, n in enumerate(NAMES):
            N = st.layers[l].w[g].rows
            a_in = st._in_of(l, g)
            a_rows = _rows_of(a_in, rows_dev)  # before the GEMM (DOWN overwrites x, QKV's input)
            dy = dy_buf[:M * N].view(M, N)
            c = st.gemm(l, g, debug_y=dy)
            torch.cuda.synchronize()
            y = dy[rows_dev].cpu().numpy()
            ref, _ = oracle.gemm(a_rows, ow[g], bias=b[n], act=nv.ACT_GELU_TANH if g == UP else 0, want_bf16=False)
            err = normwise_err(y.astype(np.float64), ref)
            worst = max(worst, err)
            assert err <= GEMM_TOL, (l, n, err)
            if g == QKV:
                assert np.array_equal(host_bits(c[rows_dev]), host_bits(dy[rows_dev].to(torch.bfloat16))), l
            # the requant of the window: bit for bit given the kernel's y (R13 i-ii) ...
            c0 = 2 * D if g == QKV else 0
            yw = np.ascontiguousarray(y[:, c0:c0 + (D if g == QKV else N)])
            a32 = np.float32(alpha[l, g])
            got = _rows_of(st._out_of(g), rows_dev)
            assert got[2] == a32
            codes, scales, _ = oracle.quantize(yw, a32)
            assert np.array_equal(got[0], codes), (l, n)
            assert np.array_equal(got[1], scales), (l, n)
            # ... and against the oracle's requant of its own fp64 y (R13, production)
            rw = np.ascontiguousarray(ref[:, c0:c0 + yw.shape[1]].astype(np.float32))
            wc, ws, _ = oracle.quantize(rw, a32)
            mm.add(got, (wc, ws))
    print(f"\n30-layer stack: worst normwise GEMM error {worst:.2e}; {mm.report()}")
    assert mm.code_diff <= 1e-3 * mm.codes and mm.zero_sign <= 1e-3 * mm.codes

    # the production forward (no debug outputs) gives the checked run's result bit for bit
    final = (host_u8(st.x.codes).copy(), host_u8(st.x.scales).copy())
    st.forward(xd)
    torch.cuda.synchronize()
    assert np.array_equal(host_u8(st.x.codes), final[0]) and np.array_equal(host_u8(st.x.scales), final[1])
