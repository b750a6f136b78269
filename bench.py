"""Throughput of the NVFP4 hot path on B200.

One step = one forward of the DiT linear stack on seeded synthetic inputs:
30 layers at 16384 tokens, hidden 3072, FFN 14336, every linear W4A4 NVFP4:
  nvfp4_quantize of the bf16 input [16384 x 3072], then per layer
  QKV 3072->9216 + bias (bf16 Q, K, V; its V third requantized in the same
  epilogue as the stand-in attention output) -> out-projection 3072->3072 +
  bias -> FFN up 3072->14336 + bias + GELU -> FFN down 14336->3072 + bias,
  each GEMM's epilogue writing the next GEMM's NVFP4 input (output tensor
  scales fixed by one calibration pass: delayed scaling).
`value` = 123.7 TFLOP of GEMM work per step / the step's device time (CUDA
events; the timed steps replayed from one CUDA graph with an event before
every launch, so per-GEMM times come from the same run).  Beside it: the
single-layer QKV workload (quantize + 4096 x 9216 x 3072 GEMM), the NVFP4 KV
cache (append, dequant of 21 slots), the 8192-token FFN pair and the next-row
kernels.  `e2e` runs the stack through the public API with host buffers.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun each rank runs the same per-GPU workload on its own GPU (weak
scaling; the path has no exchange step); rank 0 prints one JSON line with the
max-over-ranks time.  --impl reference times the CPU oracle instead (rank 0).
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

from bit_video_dit_b200 import synthetic as syn  # noqa: E402

METRIC = "W4A4 GEMM TFLOPS (% B200 FP4 peak); quantize/KV-append GB/s (% HBM peak)"
WORKLOAD = "dit_stack_30x4_16384"
FP4_OVER_BF16 = 4.0  # nominal dense FP4 / BF16 tensor throughput (9 / 2.25 PFLOP/s)
NOMINAL_FP4_TFLOPS = 9000.0
NOMINAL_HBM_GBS = 8000.0


def max_over_ranks(times: torch.Tensor, world: int) -> list[float]:
    """Each timing as the maximum over the ranks (the slowest rank sets the
    job's time).  The ranks are independent replicas; this reduction of the
    timings is the only collective of the run."""
    if world > 1:
        torch.distributed.all_reduce(times, op=torch.distributed.ReduceOp.MAX)
    return times.tolist()


def job_tflops(world: int, flops_per_rank: float, ms: float) -> float:
    """Whole-job throughput: every rank does flops_per_rank in at most ms."""
    return world * flops_per_rank / (ms * 1e-3) / 1e12


def peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": float(p["hbm_gbs"]), "bf16_tflops": float(p["bf16_tflops"]),
                "bf16_tflops_sustained": float(p.get("bf16_tflops_sustained", p["bf16_tflops"])),
                "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


class ClockSampler:
    """nvidia-smi clocks and throttle reasons, sampled during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []
        self.t = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        if self.t:
            self.t.join(timeout=2)
        sm, mx, reasons = [], 0.0, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx = max(mx, float(parts[1]))
            except ValueError:
                continue
            for name, v in zip(names, parts[3:7]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def kernel_hash(files=("common.cuh", "gemm.cu")) -> str:
    """Hash of the sources the GEMM kernel is built from."""
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "bit_video_dit_b200", "csrc")
    for f in files:
        h.update(open(os.path.join(csrc, f), "rb").read())
    return h.hexdigest()[:16]


def recorded_traffic():
    """DRAM bytes per GEMM launch of the stack (mean over a layer's four, and
    per GEMM) from the committed ncu summary, if it was taken on the current
    kernel sources."""
    path = os.path.join(ROOT, "profiles", "gemm_stack_traffic.txt")
    try:
        with open(path) as f:
            r = json.load(f)
        if r.get("kernel_hash") == kernel_hash():
            return r
    except Exception:
        pass
    return None


def measure_scale_search(nv, a, qa, ws_q, chunks, cache, ring, k_out, v_out, reps: int) -> dict:
    """ms per launch of quantize(A) and of a KV append with the scale search."""
    cache_s = nv.KVCache(cache.n_slots, cache.tokens, cache.heads, cache.head_dim, scale_search=True)
    qs = nv.empty_nvfp4(a.shape[0], a.shape[1], a.device)
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(reps)]
    nv.quantize(a, out=qs, ws=ws_q, scale_search=True)
    cache_s.append(0, *chunks[0])
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            cache.dequant(ring, k_out, v_out)
            ev[i][0].record()
            nv.quantize(a, out=qs, ws=ws_q, scale_search=True)
            ev[i][1].record()
            cache.dequant(ring, k_out, v_out)
            ev[i][2].record()
            cache_s.append(i % cache_s.n_slots, *chunks[i % len(chunks)])
            ev[i][3].record()
    g.replay()
    torch.cuda.synchronize()
    q_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    ap_ms = float(np.median([e[2].elapsed_time(e[3]) for e in ev]))
    del g
    # the fused LayerNorm + modulate + quantize of A (the step before the linear layer)
    sc = torch.randn(a.shape[1], device=a.device).mul_(0.1).to(torch.bfloat16)
    sh = torch.randn(a.shape[1], device=a.device).mul_(0.1).to(torch.bfloat16)
    ws_ln = nv.workspace(nv.OP_LN_QUANTIZE, a.shape[0], 0, a.shape[1], a.device)
    nv.ln_modulate_quantize(a, mod_scale=sc, mod_shift=sh, out=qs, ws=ws_ln)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(reps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            cache.dequant(ring, k_out, v_out)
            ev[i][0].record()
            nv.ln_modulate_quantize(a, mod_scale=sc, mod_shift=sh, out=qs, ws=ws_ln)
            ev[i][1].record()
    g.replay()
    torch.cuda.synchronize()
    ln_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    del g
    # the pages' per-chunk KV variant: K-smoothing of K, the scale search on K and V
    cache_k = nv.KVCache(cache.n_slots, cache.tokens, cache.heads, cache.head_dim, scale_search=True,
                         smooth_k=True)
    for s in range(cache_k.n_slots):
        cache_k.append(s, *chunks[s % len(chunks)])
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(reps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            cache.dequant(ring, k_out, v_out)
            ev[i][0].record()
            cache_k.append(i % cache_k.n_slots, *chunks[i % len(chunks)])
            ev[i][1].record()
            ev[i][2].record()
            cache_k.dequant(ring, k_out, v_out)
            ev[i][3].record()
    g.replay()
    torch.cuda.synchronize()
    sm_ap_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    sm_dq_ms = float(np.median([e[2].elapsed_time(e[3]) for e in ev]))
    del g
    # the keys' RoPE fused ahead of their quantize (3-frame x 22 x 40 angle table), on the
    # plain cache and on the smoothed + searched one (means of the turned keys)
    cs, sn = syn.rope_table_3d(*syn.KV_GRID, cache.head_dim)
    rope = (torch.from_numpy(cs).to(a.device), torch.from_numpy(sn).to(a.device))
    cache.append(0, *chunks[0], rope=rope)
    cache_k.append(0, *chunks[0], rope=rope)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(reps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            cache.dequant(ring, k_out, v_out)
            ev[i][0].record()
            cache.append(i % cache.n_slots, *chunks[i % len(chunks)], rope=rope)
            ev[i][1].record()
            cache.dequant(ring, k_out, v_out)
            ev[i][2].record()
            cache_k.append(i % cache_k.n_slots, *chunks[i % len(chunks)], rope=rope)
            ev[i][3].record()
    g.replay()
    torch.cuda.synchronize()
    rp_ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
    rp_sm_ms = float(np.median([e[2].elapsed_time(e[3]) for e in ev]))
    del g
    return {"quantize_ms": q_ms, "kv_append_ms": ap_ms, "ln_quantize_ms": ln_ms,
            "smooth_append_ms": sm_ap_ms, "smooth_dequant_ms": sm_dq_ms,
            "rope_append_ms": rp_ms, "rope_smooth_append_ms": rp_sm_ms}


RHT_SIGN = (1, -1, -1, 1, 1, 1, -1, 1, -1, -1, 1, -1, 1, 1, -1, -1)


def measure_ffn(nv, flush, dev, reps: int) -> dict:
    """ms per launch of the 8192-token FFN pair: quantize A [8192 x 3072], the up
    projection 3072 -> 14336 with GELU and the NVFP4 requant of its output (output
    scale from one calibration pass), and the down projection 14336 -> 3072 to bf16
    on that NVFP4 output (721.6 GFLOP each).  `flush()` evicts L2 before each
    repetition (it is captured into the timing graph)."""
    up, dn = syn.FFN_UP, syn.FFN_DOWN
    a = torch.from_numpy(syn.activations_bf16(up.M, up.K, seed=5).view(np.int16)).to(dev).view(torch.bfloat16)
    wu = torch.from_numpy(syn.normal_bf16((up.N, up.K), seed=6, std=0.02).view(np.int16)).to(dev).view(torch.bfloat16)
    wd = torch.from_numpy(syn.normal_bf16((dn.N, dn.K), seed=7, std=0.02).view(np.int16)).to(dev).view(torch.bfloat16)
    qu, qd = nv.quantize(wu), nv.quantize(wd)
    del wu, wd
    qa = nv.empty_nvfp4(up.M, up.K, dev)
    ws_q = nv.workspace(nv.OP_QUANTIZE, up.M, 0, up.K, dev)
    ws_u = nv.workspace(nv.OP_GEMM, up.M, up.N, up.K, dev)
    ws_d = nv.workspace(nv.OP_GEMM, dn.M, dn.N, dn.K, dev)
    nv.quantize(a, out=qa, ws=ws_q)
    amax = torch.zeros(1, dtype=torch.float32, device=dev)
    nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, out_amax=amax, ws=ws_u)  # calibration pass (bf16 output dropped)
    h = nv.empty_nvfp4(up.M, up.N, dev)
    h.global_scale.copy_(amax / 2688.0)
    c = torch.empty((dn.M, dn.N), dtype=torch.bfloat16, device=dev)
    nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, requant=h, bf16_out=False, ws=ws_u)
    nv.gemm(h, qd, out=c, ws=ws_d)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(4)] for _ in range(reps)]
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            flush()  # L2 flush between repetitions
            ev[i][0].record()
            nv.quantize(a, out=qa, ws=ws_q)
            ev[i][1].record()
            nv.gemm(qa, qu, act=nv.ACT_GELU_TANH, requant=h, bf16_out=False, ws=ws_u)
            ev[i][2].record()
            nv.gemm(h, qd, out=c, ws=ws_d)
            ev[i][3].record()
    g.replay()
    torch.cuda.synchronize()
    out = {k: float(np.median([e[j].elapsed_time(e[j + 1]) for e in ev]))
           for j, k in enumerate(("quantize_ms", "up_ms", "down_ms"))}
    del g
    return out


def measure_training(nv, a, w, cache, ring, k_out, v_out, reps: int) -> dict:
    """ms per launch pair of the training-side operands and the weight-gradient GEMM on
    the QKV shapes: 2D scaling of W [9216 x 3072] (both operands), the RHT transposed
    operands of X [4096 x 3072] and dY [4096 x 9216], and dW = dY^T X (231.9 GFLOP)."""
    M, K = a.shape
    N = w.shape[0]
    g = torch.Generator(device=a.device).manual_seed(77)
    dy = torch.randn((M, N), generator=g, device=a.device).to(torch.bfloat16)
    w2, w2t = nv.quantize_2d(w)
    ws2 = nv.workspace(nv.OP_QUANTIZE_2D, N, 0, K, a.device)
    xt = nv.quantize_t(a, rht_sign=RHT_SIGN)
    dyt = nv.quantize_t(dy, rht_sign=RHT_SIGN)
    wst = nv.workspace(nv.OP_QUANTIZE_T, M, 0, K, a.device)
    dw = torch.empty((N, K), dtype=torch.bfloat16, device=a.device)
    wsg = nv.workspace(nv.OP_GEMM, N, K, M, a.device)
    nv.gemm(dyt, xt, out=dw, ws=wsg)
    torch.cuda.synchronize()
    ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(8)] for _ in range(reps)]
    gr = torch.cuda.CUDAGraph()
    with torch.cuda.graph(gr):
        for i in range(reps):
            cache.dequant(ring, k_out, v_out)
            ev[i][0].record()
            nv.quantize_2d(w, out=w2, out_t=w2t, ws=ws2)
            ev[i][1].record()
            cache.dequant(ring, k_out, v_out)
            ev[i][2].record()
            nv.quantize_t(a, rht_sign=RHT_SIGN, out=xt, ws=wst)
            ev[i][3].record()
            nv.quantize_t(dy, rht_sign=RHT_SIGN, out=dyt, ws=wst)
            ev[i][4].record()
            cache.dequant(ring, k_out, v_out)
            ev[i][5].record()
            nv.gemm(dyt, xt, out=dw, ws=wsg)
            ev[i][6].record()
    gr.replay()
    torch.cuda.synchronize()
    med = lambda j: float(np.median([e[j].elapsed_time(e[j + 1]) for e in ev]))
    out = {"quantize_2d_ms": med(0), "quantize_t_x_ms": med(2), "quantize_t_dy_ms": med(3), "wgrad_ms": med(5)}
    del gr
    return out


def measure_attention(nv, cache, ring, k_out, v_out, reps: int) -> dict:
    """ms per launch of the attention of one 2640-token query chunk over the NVFP4 cache:
    all 21 slots (the set the dequant gathers) and a sink + window set of 5 slots."""
    g = torch.Generator(device=k_out.device).manual_seed(91)
    q = torch.randn((cache.tokens, cache.heads, cache.head_dim), generator=g, device=k_out.device)
    q = q.to(torch.bfloat16)
    o = torch.empty_like(q)
    ws = nv.workspace(nv.OP_KV_ATTENTION, device=k_out.device)
    chunks = nv.attention_chunks(30, 1, 24, 1, 3)  # global sink, shot sink, window of 3
    small = torch.tensor([c % cache.n_slots for c in chunks], dtype=torch.int32, device=k_out.device)
    sets = {"all": ring, "sink_window": small}
    out = {}
    for name, sl in sets.items():
        cache.attention(sl, q, out=o, ws=ws)
        torch.cuda.synchronize()
        ev = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(reps)]
        gr = torch.cuda.CUDAGraph()
        with torch.cuda.graph(gr):
            for i in range(reps):
                cache.dequant(ring, k_out, v_out)
                ev[i][0].record()
                cache.attention(sl, q, out=o, ws=ws)
                ev[i][1].record()
        gr.replay()
        torch.cuda.synchronize()
        ms = float(np.median([e[0].elapsed_time(e[1]) for e in ev]))
        keys = sl.numel() * cache.tokens
        flops = 4.0 * cache.tokens * keys * cache.head_dim * cache.heads
        out[name] = {"slots": int(sl.numel()), "keys": keys, "ms": round(ms, 4),
                     "TFLOP/s": round(flops / (ms * 1e-3) / 1e12, 1)}
        del gr
    return out


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


# --------------------------------------------------------------------------- ours
STACK_NAMES = ("qkv", "out", "up", "down")


def build_stack(nv, dev, layers: int, rank: int):
    """The 16384-token DiT linear stack with seeded N(0, 0.02) weights (the same
    generator as the parity test), its first-layer input and the calibrated
    output scales."""
    from bit_video_dit_b200.stack import LinearStack

    M, D, F = syn.STACK_M, syn.STACK_LAYER[0].K, syn.STACK_LAYER[2].N
    st = LinearStack(M, D, F, dev)
    for l in range(layers):
        w, b = syn.stack_layer_bf16(l, D, F)
        st.add_layer({k: dev_bf16(v) for k, v in w.items()}, {k: dev_bf16(v) for k, v in b.items()})
        del w
    x_host = syn.activations_bf16(M, D, seed=80 + 1000 * rank)
    x = dev_bf16(x_host)
    st.calibrate(x)
    torch.cuda.synchronize()
    return st, x, x_host


def time_stack(st, x, steps: int, warmup: int, direct: bool):
    """Warm-up steps, then `steps` timed forwards of the stack (input quantize +
    every GEMM), captured as one CUDA graph each unless `direct`.  The timed
    graph holds the launches only; a second graph of the same `steps`
    forwards, with an event before every launch (event-record nodes), gives
    the per-launch-class times (replayed apart from the timed region: each
    event pair costs a few microseconds of its own).  Returns the timed and
    the component runners, the component events and the graphs."""
    n = st.launches_per_forward()
    L = len(st.layers)
    evs = [[torch.cuda.Event(enable_timing=True, external=not direct) for _ in range(n + 1)] for _ in range(steps)]

    def fwd(ev=None):
        if ev:
            ev[0].record()
        st.quantize_input(x)
        k = 1
        for l in range(L):
            for g in range(4):
                if ev:
                    ev[k].record()
                st.gemm(l, g)
                k += 1
        if ev:
            ev[k].record()

    if direct:
        run_warm = lambda: [fwd() for _ in range(warmup)]
        run_timed = lambda: [fwd() for _ in range(steps)]
        run_comp = lambda: [fwd(evs[i]) for i in range(steps)]
        graphs = []
    else:
        gw, gt, gc = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(gw):
            for _ in range(warmup):
                fwd()
        with torch.cuda.graph(gt):
            for i in range(steps):
                fwd()
        with torch.cuda.graph(gc):
            for i in range(steps):
                fwd(evs[i])
        run_warm, run_timed, run_comp = gw.replay, gt.replay, gc.replay
        graphs = [gw, gt, gc]
    torch.cuda.synchronize()
    run_warm()
    torch.cuda.synchronize()
    return run_timed, run_comp, evs, graphs


def stack_components(evs, L: int) -> dict:
    """Mean ms per launch of the input quantize and of each GEMM of a layer."""
    q = np.mean([e[0].elapsed_time(e[1]) for e in evs])
    per = {name: [] for name in STACK_NAMES}
    for e in evs:
        k = 1
        for _ in range(L):
            for g in range(4):
                per[STACK_NAMES[g]].append(e[k].elapsed_time(e[k + 1]))
                k += 1
    return {"input_quantize": float(q), **{k: float(np.mean(v)) for k, v in per.items()}}


def measure_linear_kv(nv, dev, rank: int, steps: int, warmup: int) -> dict:
    """The single-layer and KV-cache workloads beside the stack: quantize A
    [4096 x 3072] + the QKV projection 4096 x 9216 x 3072 with bias to bf16
    (W pre-quantized once), the KV append of one 2640 x 24 x 128 K/V chunk into
    ring slot (step mod 21) and the dequant of all 21 slots, each step captured
    in a graph with events between the four launches (the 681 MB dequant output
    overwrites L2 every step)."""
    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    S, T, H, D = syn.KV_SLOTS, syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    a_host = syn.activations_bf16(M, K, seed=2 + 1000 * rank)
    w_host = syn.normal_bf16((N, K), seed=3, std=0.02)
    a = dev_bf16(a_host)
    w = dev_bf16(w_host)
    bias = dev_bf16(syn.normal_bf16((N,), seed=4, std=0.02))
    qw = nv.quantize(w)
    qa = nv.empty_nvfp4(M, K, dev)
    ws_q = nv.workspace(nv.OP_QUANTIZE, M, 0, K, dev)
    ws_g = nv.workspace(nv.OP_GEMM, M, N, K, dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    cache = nv.KVCache(S, T, H, D, dev)
    chunks = [tuple(dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, D, seed=50 + i + 1000 * rank)) for i in range(4)]
    for s_ in range(S):
        cache.append(s_, *chunks[s_ % 4])
    ring = torch.arange(S, dtype=torch.int32, device=dev)
    k_out = torch.empty((S, T, H, D), dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    nv.quantize(a, out=qa, ws=ws_q)
    nv.gemm(qa, qw, out=c, bias=bias, ws=ws_g)
    cache.dequant(ring, k_out, v_out)
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(5)] for _ in range(steps)]

    def step(i, ev=None):
        for j, f in enumerate((lambda: nv.quantize(a, out=qa, ws=ws_q),
                               lambda: nv.gemm(qa, qw, out=c, bias=bias, ws=ws_g),
                               lambda: cache.append(i % S, *chunks[i % 4]),
                               lambda: cache.dequant(ring, k_out, v_out))):
            if ev:
                ev[j].record()
            f()
        if ev:
            ev[4].record()

    gw, gt = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(gw):
        for i in range(warmup):
            step(i)
    with torch.cuda.graph(gt):
        for i in range(steps):
            step(warmup + i, evs[i])
    gw.replay()
    gt.replay()
    torch.cuda.synchronize()
    comp = np.mean([[e[j].elapsed_time(e[j + 1]) for j in range(4)] for e in evs], axis=0)
    code, _ = nv.read_device_error(ws_g)
    if code != nv.OK:
        raise RuntimeError(f"device error {code} in the QKV GEMM")
    del gw, gt
    return {"comp": comp, "a": a, "w": w, "qa": qa, "ws_q": ws_q, "chunks": chunks, "cache": cache, "ring": ring,
            "k_out": k_out, "v_out": v_out}


def e2e_stack(nv, st, x_host, steps: int) -> float:
    """ms per step of the stack through the public API with host buffers: each
    step copies its bf16 input [16384 x 3072] from pinned host memory to the
    device, runs the stack, and copies the final NVFP4 output (codes, scales,
    tensor scale) back to pinned host memory.  Copies run on their own streams
    with double-buffered device inputs, so a step's copies overlap the
    neighbouring steps' compute."""
    dev = st.device
    stream = torch.cuda.current_stream()
    x_pin = torch.from_numpy(x_host.view(np.int16)).pin_memory()
    outs = [(torch.empty(st.x.codes.shape, dtype=torch.uint8).pin_memory(),
             torch.empty(st.x.scales.shape, dtype=torch.uint8).pin_memory(),
             torch.empty(1, dtype=torch.float32).pin_memory()) for _ in range(2)]
    x_devs = [torch.empty(x_host.shape, dtype=torch.bfloat16, device=dev) for _ in range(2)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    res = [nv.empty_nvfp4(st.M, st.D, dev) for _ in range(2)]

    def run(n_steps):
        ev_in = [torch.cuda.Event() for _ in range(n_steps)]
        ev_cmp = [torch.cuda.Event() for _ in range(n_steps)]
        ev_out = [torch.cuda.Event() for _ in range(n_steps)]
        start = torch.cuda.Event(enable_timing=True)
        end = torch.cuda.Event(enable_timing=True)
        start.record(stream)
        s_in.wait_event(start)
        s_out.wait_event(start)
        for k in range(n_steps):
            b = k % 2
            with torch.cuda.stream(s_in):
                if k >= 2:
                    s_in.wait_event(ev_cmp[k - 2])
                x_devs[b].view(torch.int16).copy_(x_pin, non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if k >= 2:
                stream.wait_event(ev_out[k - 2])
            out = st.forward(x_devs[b])
            # the result leaves the stack's buffer for this step's own (the next step overwrites it)
            res[b].codes.copy_(out.codes)
            res[b].scales.copy_(out.scales)
            res[b].global_scale.copy_(out.global_scale)
            ev_cmp[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[k])
                outs[b][0].copy_(res[b].codes, non_blocking=True)
                outs[b][1].copy_(res[b].scales, non_blocking=True)
                outs[b][2].copy_(res[b].global_scale, non_blocking=True)
                ev_out[k].record(s_out)
        stream.wait_event(ev_out[n_steps - 1])
        stream.wait_event(ev_in[n_steps - 1])
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n_steps

    run(2)
    return run(steps)


def run_ours(args, rank: int, world: int) -> dict | None:
    from bit_video_dit_b200 import build as nvbuild
    from bit_video_dit_b200 import nvfp4 as nv

    nvbuild.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    L = args.layers
    st, x, x_host = build_stack(nv, dev, L, rank)
    code, _ = nv.read_device_error(st.ws_g)
    if code != nv.OK:
        raise RuntimeError(f"device error {code} during calibration")
    run_timed, run_comp, evs, graphs = time_stack(st, x, args.steps, args.warmup, args.direct)

    stream = torch.cuda.current_stream()
    clocks = ClockSampler(dev.index if dev.index is not None else 0)
    clocks.start()
    time.sleep(0.3)
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    run_timed()
    t_end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    clk = clocks.stop()
    run_comp()  # the per-launch times, apart from the timed region
    torch.cuda.synchronize()
    del graphs
    code, _ = nv.read_device_error(st.ws_g)
    if code != nv.OK:
        raise RuntimeError(f"device error {code} in the timed stack")
    total_ms = t_start.elapsed_time(t_end)
    comp = stack_components(evs, L)
    e2e_ms = e2e_stack(nv, st, x_host, max(3, min(args.steps, 10)))

    sub = None
    if not args.stack_only:
        lk = measure_linear_kv(nv, dev, rank, max(5, min(args.steps, 20)), args.warmup)
        flush = lambda: lk["cache"].dequant(lk["ring"], lk["k_out"], lk["v_out"])
        sub = {"lk": lk,
               "search": measure_scale_search(nv, lk["a"], lk["qa"], lk["ws_q"], lk["chunks"], lk["cache"],
                                              lk["ring"], lk["k_out"], lk["v_out"], reps=5),
               "train": measure_training(nv, lk["a"], lk["w"], lk["cache"], lk["ring"], lk["k_out"], lk["v_out"],
                                         reps=5),
               "attn": measure_attention(nv, lk["cache"], lk["ring"], lk["k_out"], lk["v_out"], reps=3),
               "ffn": measure_ffn(nv, flush, dev, reps=5),
               "stream": measure_codec_stream(nv, dev, rounds=4)}

    keys = ["input_quantize", *STACK_NAMES]
    times = torch.tensor([total_ms, *[comp[k] for k in keys], e2e_ms,
                          *(sub["lk"]["comp"].tolist() if sub else [0.0] * 4)], dtype=torch.float64, device=dev)
    vals = max_over_ranks(times, world)
    total_ms, e2e_ms = vals[0], vals[1 + len(keys)]
    comp = dict(zip(keys, vals[1:1 + len(keys)]))
    q2_ms, g2_ms, ap_ms, dq_ms = vals[2 + len(keys):]
    if rank != 0:
        return None
    return report(args, world, st, total_ms, comp, e2e_ms, clk, sub, (q2_ms, g2_ms, ap_ms, dq_ms))


def _rl(bound, achieved, peak, unit, **kw):
    return {"bound": bound, "achieved": round(achieved, 1), "peak": round(peak, 1), "unit": unit,
            "frac": round(achieved / peak, 4), **kw}


def report(args, world, st, total_ms, comp, e2e_ms, clk, sub, lin) -> dict:
    pk = peaks()
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
    # the stack's GEMMs run inside a long step (tens of ms, back to back, under
    # the power cap): their denominator is the sustained measured figure
    fp4_sus = pk["bf16_tflops_sustained"] * FP4_OVER_BF16
    L, M, D, F = len(st.layers), st.M, st.D, st.F
    ms_step = total_ms / args.steps
    flops = st.flops()
    value = job_tflops(world, flops, ms_step)
    shapes = {"qkv": (3 * D, D), "out": (D, D), "up": (F, D), "down": (D, F)}
    gemm_ms = sum(comp[k] for k in STACK_NAMES)  # per layer
    gemm_tflops = flops / L / (gemm_ms * 1e-3) / 1e12
    tr = recorded_traffic()
    by = {}
    for k in STACK_NAMES:
        N, K = shapes[k]
        t = 2.0 * M * N * K / (comp[k] * 1e-3) / 1e12
        g = None if tr is None else tr["per_gemm"][k]
        by[f"gemm_{k}"] = _rl("tensor", t, fp4_sus, "TFLOP/s", ms=round(comp[k], 4), shape=[M, N, K],
                              frac_of_burst=round(t / fp4_peak, 4),
                              traffic=None if g is None else g["dram_read"] + g["dram_write"])
    qbytes = M * D * 2.5625
    by["input_quantize"] = _rl("hbm", qbytes / (comp["input_quantize"] * 1e-3) / 1e9, pk["hbm_gbs"], "GB/s",
                               ms=round(comp["input_quantize"], 4))
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, fp32 accumulate); bf16 input and QKV output",
        "data": "synthetic (seeded N(0,1) activations with 0.1% x20 outlier channels, N(0,0.02) random-init "
                "weights and biases)",
        "config": {"workload": WORKLOAD, "layers": L, "M": M, "D": D, "F": F,
                   "per_layer": "QKV 3072->9216 +bias (bf16 out, V third requantized) -> out 3072->3072 +bias "
                                "requant -> up 3072->14336 +bias GELU requant -> down 14336->3072 +bias requant",
                   "step": "nvfp4_quantize of the input + 4 nvfp4_gemm per layer",
                   "parallelism": f"dp{world} (independent replicas, no collective)",
                   "l2": "inputs larger than L2: every step streams 2.1 GB of NVFP4 weights and ~10 GB of "
                         "activations through the 126 MB L2"},
        "roofline": _rl("tensor", gemm_tflops, fp4_sus, "TFLOP/s",
                        kernel="gemm_kernel (tcgen05 mxf4nvf4), all 4 GEMMs of a layer: 2*M*N*K per launch "
                               "over the launches' mean duration",
                        peak_source=f"{pk['source']} bf16 sustained x {FP4_OVER_BF16:g} (nominal FP4/BF16): the "
                                    "GEMMs run inside a long step under the power cap",
                        frac_of_burst=round(gemm_tflops / fp4_peak, 4),
                        frac_of_nominal_9pf=round(gemm_tflops / NOMINAL_FP4_TFLOPS, 4),
                        traffic=None if tr is None else tr.get("dram_bytes_per_launch")),
        "roofline_by_kernel": by,
        "components_ms": {k: round(v, 4) for k, v in comp.items()},
        "e2e": {"value": round(job_tflops(world, flops, e2e_ms), 2), "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * D * 2,
                "d2h_bytes_per_step": M * D // 2 + int(st.x.scales.numel()) + 4,
                "what": "pinned host bf16 input -> device, quantize + the 30-layer stack, final NVFP4 output "
                        "(codes, scales, tensor scale) -> pinned host, every step; copies on their own streams "
                        "(double-buffered), overlapping the neighbouring steps' compute"},
        "gpu_launches": st.launches_per_forward() * args.steps,
        "clocks": clk,
    }
    if sub:
        out.update(sub_report(sub, lin, pk, fp4_peak))
    return out


def sub_report(sub, lin, pk, fp4_peak) -> dict:
    q_ms, g_ms, ap_ms, dq_ms = lin
    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    S, T, H, D = syn.KV_SLOTS, syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    flops = 2.0 * M * N * K
    quant_bytes = M * K * 2.5625
    kv_elems = T * H * D
    append_bytes = 2 * kv_elems * 2.5625
    dequant_bytes = 2 * S * kv_elems * (0.5625 + 2.0)
    gbs = lambda b, ms: b / (ms * 1e-3) / 1e9
    search, train, attn, ffn = sub["search"], sub["train"], sub["attn"], sub["ffn"]
    up, dn = syn.FFN_UP, syn.FFN_DOWN
    return {
        "linear_4096": {
            "what": "config QKV: quantize A [4096x3072] per call + QKV GEMM 4096x9216x3072 + bias -> bf16, W "
                    "pre-quantized; graph with events, the KV dequant's 681 MB output flushing L2 every step",
            "TFLOP/s": round(flops / ((q_ms + g_ms) * 1e-3) / 1e12, 1),
            "gemm": _rl("tensor", flops / (g_ms * 1e-3) / 1e12, fp4_peak, "TFLOP/s", ms=round(g_ms, 4)),
            "quantize": _rl("hbm", gbs(quant_bytes, q_ms), pk["hbm_gbs"], "GB/s", ms=round(q_ms, 4),
                            timing="inside the step graph, events around the launch (their own ~5.5 us included)"),
            "quantize_back_to_back": _rl("hbm", gbs(quant_bytes, sub["stream"]["quantize_ms"]), pk["hbm_gbs"],
                                         "GB/s", ms=round(sub["stream"]["quantize_ms"], 4),
                                         timing="32 launches back to back over 8 rotating 25 MB inputs (201 MB > "
                                                "L2), one pair of events"),
            "quantize_given_scale_back_to_back": _rl(
                "hbm", gbs(quant_bytes, sub["stream"]["quantize_given_scale_ms"]), pk["hbm_gbs"], "GB/s",
                ms=round(sub["stream"]["quantize_given_scale_ms"], 4),
                timing="as quantize_back_to_back, the tensor scale given (NVFP4_Q_GIVEN_GLOBAL, delayed scaling: "
                       "no grid-wide maximum, so the encode overlaps the loads)")},
        "kv": {
            "what": "NVFP4 KV cache of 21 slots x 2640 x 24 x 128: append of one K/V chunk (in place into ring "
                    "slot step mod 21), dequant-gather of all 21 slots to bf16",
            "append": _rl("hbm", gbs(append_bytes, ap_ms), pk["hbm_gbs"], "GB/s", ms=round(ap_ms, 4),
                          timing="inside the step graph, events around the launch (their own ~5.5 us included)"),
            "append_back_to_back": _rl("hbm", gbs(append_bytes, sub["stream"]["kv_append_ms"]), pk["hbm_gbs"],
                                       "GB/s", ms=round(sub["stream"]["kv_append_ms"], 4),
                                       timing="32 appends back to back over 8 rotating 32 MB K/V chunks (260 MB > "
                                              "L2) into 8 slots, one pair of events"),
            "dequant": _rl("hbm", gbs(dequant_bytes, dq_ms), pk["hbm_gbs"], "GB/s", ms=round(dq_ms, 4)),
            "cache_bytes": sub["lk"]["cache"].nbytes()},
        "scale_search": {
            "what": "adaptive per-block scale search over the targets {4, 6}",
            "quantize_ms": round(search["quantize_ms"], 4),
            "quantize_GB/s": round(gbs(quant_bytes, search["quantize_ms"]), 1),
            "kv_append_ms": round(search["kv_append_ms"], 4),
            "kv_append_GB/s": round(gbs(append_bytes, search["kv_append_ms"]), 1)},
        "kv_smoothing": {
            "what": "KV append with K-smoothing of K and the scale search on K and V (channel means + quantize), "
                    "and the dequant of all slots with the means added back",
            "append_ms": round(search["smooth_append_ms"], 4),
            "append_GB/s": round(gbs(append_bytes, search["smooth_append_ms"]), 1),
            "dequant_ms": round(search["smooth_dequant_ms"], 4),
            "dequant_GB/s": round(gbs(dequant_bytes, search["smooth_dequant_ms"]), 1)},
        "kv_rope": {
            "what": "KV append with the keys' rotary embedding fused ahead of their quantize (3-frame x 22 x 40 "
                    "angle table), plain and with K-smoothing + scale search; GB/s of the append's bytes",
            "append_ms": round(search["rope_append_ms"], 4),
            "append_GB/s": round(gbs(append_bytes, search["rope_append_ms"]), 1),
            "smooth_search_append_ms": round(search["rope_smooth_append_ms"], 4),
            "smooth_search_append_GB/s": round(gbs(append_bytes, search["rope_smooth_append_ms"]), 1)},
        "ffn_8192": {
            "what": "config FFN: quantize A [8192x3072], up 3072->14336 with GELU and the NVFP4 requant of its "
                    "output, down 14336->3072 to bf16 on that output; each 2*M*N*K = 721.6 GFLOP",
            "quantize_ms": round(ffn["quantize_ms"], 4),
            "up": _rl("tensor", 2 * up.M * up.N * up.K / (ffn["up_ms"] * 1e-3) / 1e12, fp4_peak, "TFLOP/s",
                      ms=round(ffn["up_ms"], 4)),
            "down": _rl("tensor", 2 * dn.M * dn.N * dn.K / (ffn["down_ms"] * 1e-3) / 1e12, fp4_peak, "TFLOP/s",
                        ms=round(ffn["down_ms"], 4))},
        "training": {
            "what": "training-side NVFP4 on the QKV layer shapes: 2D (16x16) scaling of W [9216x3072] writing W "
                    "and W^T operands; RHT + transposed 1D quantize of X [4096x3072] and dY [4096x9216]; "
                    "dW = dY^T X (9216x3072x4096) on those operands",
            "quantize_2d_ms": round(train["quantize_2d_ms"], 4),
            "quantize_2d_GB/s": round(gbs(N * K * 3.125, train["quantize_2d_ms"]), 1),
            "quantize_t_x_ms": round(train["quantize_t_x_ms"], 4),
            "quantize_t_x_GB/s": round(gbs(M * K * 2.5625, train["quantize_t_x_ms"]), 1),
            "quantize_t_dy_ms": round(train["quantize_t_dy_ms"], 4),
            "quantize_t_dy_GB/s": round(gbs(M * N * 2.5625, train["quantize_t_dy_ms"]), 1),
            "wgrad_ms": round(train["wgrad_ms"], 4),
            "wgrad_TFLOP/s": round(2.0 * N * K * M / (train["wgrad_ms"] * 1e-3) / 1e12, 1)},
        "kv_attention": {
            "what": "softmax attention of one 2640x24x128 bf16 query chunk over NVFP4 cache slots read directly; "
                    "TFLOP/s counts 4*Tq*keys*d*H", "bf16_peak_TFLOP/s": pk.get("bf16_tflops"), **attn},
        "ln_modulate_quantize": {
            "what": "LayerNorm + adaLN modulate + NVFP4 quantize of A [4096x3072]",
            "ms": round(search["ln_quantize_ms"], 4),
            "GB/s": round(gbs(quant_bytes, search["ln_quantize_ms"]), 1),
            "back_to_back_ms": round(sub["stream"]["ln_quantize_ms"], 4),
            "back_to_back_GB/s": round(gbs(quant_bytes, sub["stream"]["ln_quantize_ms"]), 1)},
    }


def measure_codecs(nv, dev, reps: int) -> dict:
    """ms per launch (median over `reps`, each after a 256 MB L2 flush, inside
    one graph) of the codec kernels on their workloads: quantize of A
    [4096 x 3072], the KV append of one 2640 x 24 x 128 K/V chunk, the dequant
    of 21 slots, and the LayerNorm + modulate + quantize of A.  Also the small
    case for profiling those kernels (under 2 GB on the device)."""
    M, K = syn.QKV.M, syn.QKV.K
    S, T, H, D = syn.KV_SLOTS, syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    a = dev_bf16(syn.activations_bf16(M, K, seed=2))
    qa = nv.empty_nvfp4(M, K, dev)
    ws_q = nv.workspace(nv.OP_QUANTIZE, M, 0, K, dev)
    ws_ln = nv.workspace(nv.OP_LN_QUANTIZE, M, 0, K, dev)
    sc = dev_bf16(syn.normal_bf16((K,), seed=72, std=0.1))
    sh = dev_bf16(syn.normal_bf16((K,), seed=73, std=0.1))
    cache = nv.KVCache(S, T, H, D, dev)
    k, v = (dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, D, seed=50))
    for s_ in range(S):
        cache.append(s_, k, v)
    ring = torch.arange(S, dtype=torch.int32, device=dev)
    k_out = torch.empty((S, T, H, D), dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    flush = torch.empty(256 << 20, dtype=torch.uint8, device=dev)
    calls = {"quantize_ms": lambda: nv.quantize(a, out=qa, ws=ws_q),
             "kv_append_ms": lambda: cache.append(0, k, v),
             "kv_dequant_ms": lambda: cache.dequant(ring, k_out, v_out),
             "ln_quantize_ms": lambda: nv.ln_modulate_quantize(a, mod_scale=sc, mod_shift=sh, out=qa, ws=ws_ln)}
    for f in calls.values():
        f()
    torch.cuda.synchronize()
    ev = {name: [[torch.cuda.Event(enable_timing=True, external=True) for _ in range(2)] for _ in range(reps)]
          for name in calls}
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        for i in range(reps):
            for name, f in calls.items():
                flush.fill_(1)
                ev[name][i][0].record()
                f()
                ev[name][i][1].record()
    g.replay()
    torch.cuda.synchronize()
    out = {name: float(np.median([e[0].elapsed_time(e[1]) for e in evs])) for name, evs in ev.items()}
    del g
    return out


def measure_codec_stream(nv, dev, rounds: int) -> dict:
    """ms per launch of the codec kernels launched back to back inside one
    graph, every launch on its own buffers from a set larger than L2 (8 copies
    of A [4096 x 3072], 201 MB; 8 K/V chunk pairs, 260 MB; the outputs rotate
    too), so each launch reads its inputs from HBM; one pair of events brackets
    `rounds` x 8 launches, so the events' own cost per kernel (~5.5 us here
    between two events around even a one-element kernel) is not charged to
    each launch, only the gaps between launches."""
    M, K = syn.QKV.M, syn.QKV.K
    T, H, D = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    nb = 8
    a0 = dev_bf16(syn.activations_bf16(M, K, seed=2))
    acts = [a0.clone() for _ in range(nb)]
    outs = [nv.empty_nvfp4(M, K, dev) for _ in range(nb)]
    ws_q = nv.workspace(nv.OP_QUANTIZE, M, 0, K, dev)
    ws_ln = nv.workspace(nv.OP_LN_QUANTIZE, M, 0, K, dev)
    sc = dev_bf16(syn.normal_bf16((K,), seed=72, std=0.1))
    sh = dev_bf16(syn.normal_bf16((K,), seed=73, std=0.1))
    k0, v0 = (dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, D, seed=50))
    chunks = [(k0.clone(), v0.clone()) for _ in range(nb)]
    cache = nv.KVCache(nb, T, H, D, dev)
    given = torch.empty(1, dtype=torch.float32, device=dev)
    nv.quantize(acts[0], out=outs[0], ws=ws_q)
    given.copy_(outs[0].global_scale)
    calls = {"quantize_ms": lambda i: nv.quantize(acts[i], out=outs[i], ws=ws_q),
             "quantize_given_scale_ms": lambda i: nv.quantize(acts[i], global_scale=given, out=outs[i], ws=ws_q),
             "kv_append_ms": lambda i: cache.append(i, *chunks[i]),
             "ln_quantize_ms": lambda i: nv.ln_modulate_quantize(acts[i], mod_scale=sc, mod_shift=sh, out=outs[i],
                                                                 ws=ws_ln)}
    out = {}
    for name, f in calls.items():
        for i in range(nb):
            f(i)
        torch.cuda.synchronize()
        e0 = torch.cuda.Event(enable_timing=True, external=True)
        e1 = torch.cuda.Event(enable_timing=True, external=True)
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g):
            e0.record()
            for _ in range(rounds):
                for i in range(nb):
                    f(i)
            e1.record()
        g.replay()
        torch.cuda.synchronize()
        g.replay()
        torch.cuda.synchronize()
        out[name] = e0.elapsed_time(e1) / (rounds * nb)
        del g
    return out


# --------------------------------------------------------------------------- oracle
def _timed(f):
    t0 = time.perf_counter()
    f()
    return time.perf_counter() - t0


def oracle_stack_rows(rows: int, layer_w, x_rows_bits):
    """The oracle on `rows` token rows through one layer of the stack: the
    quantize of those input rows, then the four fp64 GEMMs with their epilogues
    and the binary32 requants between them (output scales from the rows
    themselves).  Returns seconds."""
    import oracle

    def run():
        codes, scales, a32 = oracle.quantize(x_rows_bits)
        a = (codes, scales, a32)
        D = x_rows_bits.shape[1]
        for g, (w, b) in enumerate(layer_w):
            y, _ = oracle.gemm(a, w, bias=b, act=1 if g == 2 else 0, want_bf16=False)
            if g == 0:
                y = y[:, 2 * D:]
            y = np.ascontiguousarray(y.astype(np.float32))
            a = oracle.quantize(y)
    return _timed(run)


def oracle_layer_weights(layer: int):
    import oracle

    D, F = syn.STACK_LAYER[0].K, syn.STACK_LAYER[2].N
    w, b = syn.stack_layer_bf16(layer, D, F)
    return [(oracle.quantize(w[n]), b[n]) for n in STACK_NAMES]


def cpu_baseline(rows: int = 4) -> dict:
    """The oracle on the host cores: the stack's rate on `rows` token rows of
    one layer (the headline's sample, extrapolated to the full stack), and the
    codec work of the KV workload and the activation quantize timed in full."""
    import oracle

    D = syn.STACK_LAYER[0].K
    lw = oracle_layer_weights(0)
    x = syn.activations_bf16(rows, D, seed=80)
    t = oracle_stack_rows(rows, lw, x)
    per_row = 2.0 * (3 * D * D + D * D + 2 * syn.STACK_LAYER[2].N * D)
    value = rows * per_row / t / 1e12
    full_stack_s = syn.STACK_LAYERS * syn.STACK_M * per_row / (value * 1e12)
    # codec work in full: quantize of A [4096 x 3072], a KV append of one chunk, the dequant of 21 slots
    M, K = syn.QKV.M, syn.QKV.K
    a = syn.activations_bf16(M, K, seed=2)
    tq = _timed(lambda: oracle.quantize(a))
    T, H, Dh = syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
    k, v = syn.kv_chunk_bf16(T, H, Dh, seed=50)
    res = {}
    ta = _timed(lambda: res.update(k=oracle.kv_append(k), v=oracle.kv_append(v)))
    td = _timed(lambda: [oracle.kv_dequant(*res["k"], T, H, Dh) for _ in range(syn.KV_SLOTS)] +
                [oracle.kv_dequant(*res["v"], T, H, Dh) for _ in range(syn.KV_SLOTS)])
    kv_elems = T * H * Dh
    gemms = oracle_gemm_configs(rows=8)
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(), "kind": "oracle",
            "host_cores": os.cpu_count(),
            "sample": f"{rows} of {syn.STACK_M} token rows through one layer of the stack (input quantize, 4 fp64 "
                      "GEMMs with epilogues, 4 binary32 requants)",
            "extrapolated_full_stack_s": round(full_stack_s, 1),
            "codecs_in_full": {
                "quantize_4096x3072_GB/s": round(M * K * 2.5625 / tq / 1e9, 4),
                "kv_append_GB/s": round(2 * kv_elems * 2.5625 / ta / 1e9, 4),
                "kv_dequant_21_slots_GB/s": round(2 * syn.KV_SLOTS * kv_elems * 2.5625 / td / 1e9, 4),
                "seconds": round(tq + ta + td, 2)},
            "gemm_configs": gemms}


def oracle_gemm_configs(rows: int) -> dict:
    """The oracle's fp64 GEMM (with its epilogue) per configuration: the tiny
    64 x 128 x 256 case in full, the QKV projection and the FFN pair on `rows`
    token rows (the weights quantized in full by the oracle first), with the
    full-size time extrapolated from the rows' rate."""
    import oracle

    out = {}
    a = syn.tiny_a_bf16(64, 256, seed=0)
    w = syn.normal_bf16((128, 256), seed=1)
    qa, qw = oracle.quantize(a), oracle.quantize(w)
    t = _timed(lambda: oracle.gemm(qa, qw, want_bf16=True))
    out["tiny_64x128x256_full"] = {"TFLOP/s": round(2.0 * 64 * 128 * 256 / t / 1e12, 6), "seconds": round(t, 4)}
    shapes = {"qkv_4096x9216x3072": (syn.QKV, 0), "ffn_up_8192x14336x3072": (syn.FFN_UP, nv_act_gelu()),
              "ffn_down_8192x3072x14336": (syn.FFN_DOWN, 0)}
    for name, (sh, act) in shapes.items():
        x = syn.activations_bf16(rows, sh.K, seed=2)
        wq = oracle.quantize(syn.normal_bf16_blocks((sh.N, sh.K), seed=3, std=0.02))
        bias = syn.normal_bf16((sh.N,), seed=4, std=0.02)
        xq = oracle.quantize(x)
        t = _timed(lambda: oracle.gemm(xq, wq, bias=bias, act=act, want_bf16=True))
        rate = 2.0 * rows * sh.N * sh.K / t
        out[name] = {"rows": rows, "TFLOP/s": round(rate / 1e12, 6),
                     "extrapolated_full_s": round(2.0 * sh.M * sh.N * sh.K / rate, 1)}
    return out


def nv_act_gelu() -> int:
    from bit_video_dit_b200 import nvfp4 as nv

    return nv.ACT_GELU_TANH


def run_reference(args) -> dict:
    """--impl reference: the oracle, as it stands, on the stack's metric: each
    step one layer (cycling over two seeded layers) on a few token rows."""
    import oracle

    D = syn.STACK_LAYER[0].K
    rows = 4
    lws = [oracle_layer_weights(l) for l in range(2)]
    x = syn.activations_bf16(rows, D, seed=80)
    for i in range(args.warmup):
        oracle_stack_rows(rows, lws[i % 2], x)
    t = sum(oracle_stack_rows(rows, lws[i % 2], x) for i in range(args.steps))
    per_row = 2.0 * (3 * D * D + D * D + 2 * syn.STACK_LAYER[2].N * D)
    value = args.steps * rows * per_row / t / 1e12
    sample = (f"{rows} of {syn.STACK_M} token rows through one layer of the stack per step (layers 0 and 1 in turn): "
              "input quantize, 4 fp64 GEMMs with epilogues, 4 binary32 requants")
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 GEMM over NVFP4 operands; f32 quantize",
            "data": "synthetic (seeded, same generators as the GPU arm)", "impl": "reference",
            "config": {"workload": WORKLOAD, "layers": syn.STACK_LAYERS, "M": syn.STACK_M,
                       "parallelism": "cpu oracle, rank 0"},
            "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(),
                             "kind": "oracle", "sample": sample},
            "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


def main(argv=None) -> int:
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--direct", action="store_true",
                    help="launch each component on the stream instead of replaying it from a CUDA graph")
    ap.add_argument("--ffn-only", action="store_true",
                    help="time only the 8192-token FFN pair (under 1 GB on the device: the small case for "
                         "profiling its GEMMs) and print its numbers")
    ap.add_argument("--codecs-only", action="store_true",
                    help="time only the codec kernels (quantize, KV append / dequant, LayerNorm quantize) on their "
                         "workloads and print their numbers (also the small case for profiling them)")
    ap.add_argument("--layers", type=int, default=syn.STACK_LAYERS,
                    help="layers of the stack (default 30, the workload; fewer only for profiling)")
    ap.add_argument("--attention-only", action="store_true",
                    help="time only the attention over the KV workload's 21-slot cache (about 1 GB on the device: "
                         "the case for profiling the attention kernel) and print its numbers")
    ap.add_argument("--stack-only", action="store_true",
                    help="time the stack alone (skip the single-layer, KV and next-row measurements)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))

    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return 0

    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (there is no CPU fallback)")
    torch.cuda.set_device(local)
    if args.ffn_only:
        from bit_video_dit_b200 import build as nvbuild
        from bit_video_dit_b200 import nvfp4 as nv
        nvbuild.build()
        flush_buf = torch.empty(256 << 20, dtype=torch.uint8, device="cuda")  # 256 MB > L2
        ffn = measure_ffn(nv, lambda: flush_buf.fill_(1), flush_buf.device, reps=max(1, args.steps))
        if rank == 0:
            print(json.dumps({"ffn_8192": {k: round(v, 4) for k, v in ffn.items()}}), flush=True)
        return 0
    if args.attention_only:
        from bit_video_dit_b200 import build as nvbuild
        from bit_video_dit_b200 import nvfp4 as nv
        nvbuild.build()
        dev = torch.device("cuda", local)
        S, T, H, D = syn.KV_SLOTS, syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM
        cache = nv.KVCache(S, T, H, D, dev)
        chunks = [tuple(dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, D, seed=50 + i)) for i in range(4)]
        for s_ in range(S):
            cache.append(s_, *chunks[s_ % 4])
        ring = torch.arange(S, dtype=torch.int32, device=dev)
        k_out = torch.empty((S, T, H, D), dtype=torch.bfloat16, device=dev)
        v_out = torch.empty_like(k_out)
        res = measure_attention(nv, cache, ring, k_out, v_out, reps=max(3, args.steps))
        if rank == 0:
            print(json.dumps({"kv_attention": res, "bf16_peak_TFLOP/s": peaks()["bf16_tflops"]}), flush=True)
        return 0
    if args.codecs_only:
        from bit_video_dit_b200 import build as nvbuild
        from bit_video_dit_b200 import nvfp4 as nv
        nvbuild.build()
        dev = torch.device("cuda", local)
        res = measure_codecs(nv, dev, reps=max(3, args.steps))
        stream_res = measure_codec_stream(nv, dev, rounds=max(2, args.steps))
        pk = peaks()
        b = {"quantize_ms": syn.QKV.M * syn.QKV.K * 2.5625, "ln_quantize_ms": syn.QKV.M * syn.QKV.K * 2.5625,
             "quantize_given_scale_ms": syn.QKV.M * syn.QKV.K * 2.5625,
             "kv_append_ms": 2 * syn.KV_TOKENS * syn.KV_HEADS * syn.KV_DIM * 2.5625,
             "kv_dequant_ms": 2 * syn.KV_SLOTS * syn.KV_TOKENS * syn.KV_HEADS * syn.KV_DIM * 2.5625}
        line = lambda r: {k: {"ms": round(v, 4), "GB/s": round(b[k] / (v * 1e-3) / 1e9, 1),
                              "frac_hbm": round(b[k] / (v * 1e-3) / 1e9 / pk["hbm_gbs"], 4)} for k, v in r.items()}
        if rank == 0:
            print(json.dumps({"flushed_each": line(res), "back_to_back": line(stream_res)}), flush=True)
        return 0
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        out = run_ours(args, rank, world)
        if rank == 0 and out is not None:
            if not args.no_cpu_baseline and world == 1:
                out["cpu_baseline"] = cpu_baseline()
            if args.layers != syn.STACK_LAYERS:
                out["config"]["workload"] = f"dit_stack_{args.layers}x4_16384 (reduced: not the workload)"
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
