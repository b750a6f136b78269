"""Throughput of the NVFP4 hot path on B200.

One step = one pass of the whole path on seeded synthetic DiT-shaped inputs:
  1. nvfp4_quantize  of the activation A [4096 x 3072] bf16 (tensor amax,
     block scales, E2M1 codes, swizzled scale tiles)
  2. nvfp4_gemm      QKV projection 4096 x 9216 x 3072, W pre-quantized once,
     bias epilogue, bf16 out
  3. nvfp4_kv_append of one frame-chunk's K and V [2640 x 24 x 128] into ring
     slot step % 21
  4. nvfp4_kv_dequant of all 21 slots (ring order) back to bf16
`value` is the W4A4 linear-layer throughput (2*M*N*K of step 2 per second of
steps 1+2, device-timed with CUDA events); the KV rows are reported under
"kv".  The timed steps are captured as one CUDA graph, with the timing events
between components as event-record nodes, so the timed region holds device
work only (no host launch gaps); `e2e` instead
calls the public Python API with host buffers every step.  The 681 MB bf16 output of step 4 overwrites L2 (126 MB) every step, so
each step's GEMM and quantize read their inputs from HBM.

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
WORKLOAD = "dit_qkv_4096x9216x3072_bias+kv_append_dequant_21x2640x24x128"
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
    """DRAM bytes per GEMM launch from the committed ncu summary, if it was
    taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "gemm_qkv_traffic.txt")
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
def run_ours(args, rank: int, world: int) -> dict | None:
    from bit_video_dit_b200 import build as nvbuild
    from bit_video_dit_b200 import nvfp4 as nv

    nvbuild.build()
    dev = torch.device("cuda", torch.cuda.current_device())
    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    S, T, H, D = syn.KV_SLOTS, syn.KV_TOKENS, syn.KV_HEADS, syn.KV_DIM

    a_host = syn.activations_bf16(M, K, seed=2 + 1000 * rank)
    w_host = syn.normal_bf16((N, K), seed=3, std=0.02)
    bias_host = syn.normal_bf16((N,), seed=4, std=0.02)
    a = dev_bf16(a_host)
    w = dev_bf16(w_host)
    bias = dev_bf16(bias_host)
    qw = nv.quantize(w)  # weights quantized once
    del w
    qa = nv.empty_nvfp4(M, K, dev)
    ws_q = nv.workspace(nv.OP_QUANTIZE, M, 0, K, dev)
    ws_g = nv.workspace(nv.OP_GEMM, M, N, K, dev)
    c = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    cache = nv.KVCache(S, T, H, D, dev)
    n_chunks = 4  # distinct K/V chunks cycled through the ring
    chunks = [tuple(dev_bf16(x) for x in syn.kv_chunk_bf16(T, H, D, seed=50 + i + 1000 * rank))
              for i in range(n_chunks)]
    for s in range(S):
        cache.append(s, *chunks[s % n_chunks])
    ring = torch.arange(S, dtype=torch.int32, device=dev)
    k_out = torch.empty((S, T, H, D), dtype=torch.bfloat16, device=dev)
    v_out = torch.empty_like(k_out)
    stream = torch.cuda.current_stream()

    do_quant = lambda: nv.quantize(a, out=qa, ws=ws_q)
    do_gemm = lambda: nv.gemm(qa, qw, out=c, bias=bias, ws=ws_g)
    do_append = [lambda s=s: cache.append(s, *chunks[s % n_chunks]) for s in range(S)]
    do_dequant = lambda: cache.dequant(ring, k_out, v_out)
    for f in (do_quant, do_gemm, do_append[0], do_dequant):
        f()  # first calls set kernel attributes and resolve the driver entry point
    torch.cuda.synchronize()

    def step(i, ev=None):
        if ev:
            ev[0].record()  # the current (capture) stream
        do_quant()
        if ev:
            ev[1].record()  # the current (capture) stream
        do_gemm()
        if ev:
            ev[2].record()  # the current (capture) stream
        do_append[i % S]()
        if ev:
            ev[3].record()  # the current (capture) stream
        do_dequant()
        if ev:
            ev[4].record()  # the current (capture) stream

    # By default the warm-up steps and the timed steps are each captured as one
    # CUDA graph (the timing events between the components become event-record
    # nodes), so the timed region holds device work only: no host launch gaps
    # and no per-component graph launches.  --direct launches every component
    # on the stream instead.
    evs = [[torch.cuda.Event(enable_timing=True, external=not args.direct) for _ in range(5)]
           for _ in range(args.steps)]
    if args.direct:
        run_warmup = lambda: [step(i) for i in range(args.warmup)]
        run_timed = lambda: [step(args.warmup + i, evs[i]) for i in range(args.steps)]
        graphs = []
    else:
        g_warm, g_timed = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
        with torch.cuda.graph(g_warm):
            for i in range(args.warmup):
                step(i)
        with torch.cuda.graph(g_timed):
            for i in range(args.steps):
                step(args.warmup + i, evs[i])
        run_warmup, run_timed = g_warm.replay, g_timed.replay
        graphs = [g_warm, g_timed]
    torch.cuda.synchronize()

    run_warmup()
    torch.cuda.synchronize()
    code, _ = nv.read_device_error(ws_g)
    if code != nv.OK:
        raise RuntimeError(f"device error {code} during warm-up")

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
    del graphs

    # The adaptive scale search ({4, 6}) variants of the two quantize launches,
    # timed the same way (inside a graph, each after a dequant of all slots so
    # that its input comes from HBM); reported beside the step, not part of it.
    search = measure_scale_search(nv, a, qa, ws_q, chunks, cache, ring, k_out, v_out, reps=5)
    # the training-side operands (2D weight scaling, RHT transposed operands) and the
    # weight-gradient GEMM on the same layer shapes, also beside the step
    train = measure_training(nv, a, dev_bf16(w_host), cache, ring, k_out, v_out, reps=5)
    # attention reading the NVFP4 cache directly (one query chunk), beside the step
    attn = measure_attention(nv, cache, ring, k_out, v_out, reps=3)
    # the 8192-token FFN pair (up with GELU + requant, down to bf16), beside the step
    ffn = measure_ffn(nv, lambda: cache.dequant(ring, k_out, v_out), k_out.device, reps=5)

    total_ms = t_start.elapsed_time(t_end)
    comp = np.zeros(4)
    for e in evs:
        comp += [e[j].elapsed_time(e[j + 1]) for j in range(4)]
    comp /= args.steps  # ms per step per component: quantize, gemm, append, dequant

    # --- e2e through the public API with host buffers (linear layer) -------
    # Every step copies its own A from pinned host memory and its C back to
    # pinned host memory inside the timed region.  The copies run on their own
    # streams with double-buffered device tensors, so step k+1's host->device
    # copy and step k-1's device->host copy overlap step k's compute (PCIe is
    # full duplex: one copy engine per direction).
    a_pin = torch.from_numpy(a_host.view(np.int16)).pin_memory()
    c_pins = [torch.empty((M, N), dtype=torch.int16).pin_memory() for _ in range(2)]
    a_devs = [torch.empty((M, K), dtype=torch.bfloat16, device=dev) for _ in range(2)]
    c_devs = [c, torch.empty_like(c)]
    s_in, s_out = torch.cuda.Stream(device=dev), torch.cuda.Stream(device=dev)
    e2e_steps = max(3, min(args.steps, 10))

    def e2e_run(n_steps):
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
                    s_in.wait_event(ev_cmp[k - 2])  # a_devs[b] is free once step k-2 has read it
                a_devs[b].view(torch.int16).copy_(a_pin, non_blocking=True)
                ev_in[k].record(s_in)
            stream.wait_event(ev_in[k])
            if k >= 2:
                stream.wait_event(ev_out[k - 2])  # c_devs[b] is free once step k-2's result is on the host
            nv.quantize(a_devs[b], out=qa, ws=ws_q)
            nv.gemm(qa, qw, out=c_devs[b], bias=bias, ws=ws_g)
            ev_cmp[k].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_cmp[k])
                c_pins[b].copy_(c_devs[b].view(torch.int16), non_blocking=True)
                ev_out[k].record(s_out)
        stream.wait_event(ev_out[n_steps - 1])
        stream.wait_event(ev_in[n_steps - 1])
        end.record(stream)
        torch.cuda.synchronize()
        return start.elapsed_time(end) / n_steps

    e2e_run(2)
    e2e_ms = e2e_run(e2e_steps)

    times = torch.tensor([total_ms, *comp.tolist(), e2e_ms], dtype=torch.float64, device=dev)
    total_ms, q_ms, g_ms, ap_ms, dq_ms, e2e_ms = max_over_ranks(times, world)
    if rank != 0:
        return None

    pk = peaks()
    flops = 2.0 * M * N * K
    lin_ms = q_ms + g_ms
    value = job_tflops(world, flops, lin_ms)
    gemm_tflops = flops / (g_ms * 1e-3) / 1e12
    fp4_peak = pk["bf16_tflops"] * FP4_OVER_BF16
    quant_bytes = M * K * 2.5625
    kv_elems = T * H * D
    append_bytes = 2 * kv_elems * 2.5625
    dequant_bytes = 2 * S * kv_elems * (0.5625 + 2.0)
    tr = recorded_traffic()
    out = {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 4),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "nvfp4 (e2m1 x e2m1, e4m3 block scales, fp32 accumulate); bf16 in/out",
        "data": "synthetic (seeded N(0,1) activations with 0.1% x20 outlier channels, N(0,0.02) weights)",
        "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "kv_slots": S, "kv_tokens": T, "kv_heads": H,
                   "kv_head_dim": D, "parallelism": f"dp{world} (independent replicas, no collective)",
                   "l2": "inputs larger than L2: each step's 681 MB KV dequant output overwrites the 126 MB L2"},
        "roofline": {"kernel": "nvfp4 gemm (tcgen05 mxf4nvf4)", "bound": "tensor",
                     "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1), "unit": "TFLOP/s",
                     "frac": round(gemm_tflops / fp4_peak, 4),
                     "peak_source": f"{pk['source']} bf16 burst x {FP4_OVER_BF16:g} (nominal FP4/BF16)",
                     "frac_of_nominal_9pf": round(gemm_tflops / NOMINAL_FP4_TFLOPS, 4),
                     "traffic": None if tr is None else tr["dram_bytes_per_launch"],
                     "algorithmic_bytes": M * K // 2 + N * K // 2 + (M + N) * K // 16 + M * N * 2},
        "roofline_by_kernel": {
            "gemm": {"bound": "tensor", "achieved": round(gemm_tflops, 1), "peak": round(fp4_peak, 1),
                     "unit": "TFLOP/s", "frac": round(gemm_tflops / fp4_peak, 4)},
            "quantize": {"bound": "hbm", "achieved": round(quant_bytes / (q_ms * 1e-3) / 1e9, 1),
                         "peak": pk["hbm_gbs"], "unit": "GB/s",
                         "frac": round(quant_bytes / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
            "kv_append": {"bound": "hbm", "achieved": round(append_bytes / (ap_ms * 1e-3) / 1e9, 1),
                          "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": round(append_bytes / (ap_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)},
            "kv_dequant": {"bound": "hbm", "achieved": round(dequant_bytes / (dq_ms * 1e-3) / 1e9, 1),
                           "peak": pk["hbm_gbs"], "unit": "GB/s",
                           "frac": round(dequant_bytes / (dq_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4)}},
        "components_ms": {"quantize": round(q_ms, 4), "gemm": round(g_ms, 4), "kv_append": round(ap_ms, 4),
                          "kv_dequant": round(dq_ms, 4)},
        "quantize": {"GB/s": round(quant_bytes / (q_ms * 1e-3) / 1e9, 1),
                     "frac_hbm": round(quant_bytes / (q_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
                     "bytes_per_call": quant_bytes},
        "kv": {"append_GB/s": round(append_bytes / (ap_ms * 1e-3) / 1e9, 1),
               "append_frac_hbm": round(append_bytes / (ap_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
               "dequant_GB/s": round(dequant_bytes / (dq_ms * 1e-3) / 1e9, 1),
               "dequant_frac_hbm": round(dequant_bytes / (dq_ms * 1e-3) / 1e9 / pk["hbm_gbs"], 4),
               "hbm_peak_GB/s": pk["hbm_gbs"], "cache_bytes": cache.nbytes()},
        "scale_search": {
            "what": "adaptive per-block scale search over the targets {4, 6}, outside the step",
            "quantize_ms": round(search["quantize_ms"], 4),
            "quantize_GB/s": round(quant_bytes / (search["quantize_ms"] * 1e-3) / 1e9, 1),
            "kv_append_ms": round(search["kv_append_ms"], 4),
            "kv_append_GB/s": round(append_bytes / (search["kv_append_ms"] * 1e-3) / 1e9, 1)},
        "kv_smoothing": {
            "what": "KV append with K-smoothing of K and the scale search on K and V (channel means + quantize, "
                    "two launches), and the dequant of all slots with the means added back, outside the step",
            "append_ms": round(search["smooth_append_ms"], 4),
            "append_GB/s": round(append_bytes / (search["smooth_append_ms"] * 1e-3) / 1e9, 1),
            "dequant_ms": round(search["smooth_dequant_ms"], 4),
            "dequant_GB/s": round(dequant_bytes / (search["smooth_dequant_ms"] * 1e-3) / 1e9, 1)},
        "kv_rope": {
            "what": "KV append with the keys' rotary embedding fused ahead of their quantize (3-frame x 22 x 40 "
                    "angle table read from L2), plain and with K-smoothing + scale search (means of the turned "
                    "keys, two launches), outside the step; GB/s counts the append's algorithmic bytes",
            "append_ms": round(search["rope_append_ms"], 4),
            "append_GB/s": round(append_bytes / (search["rope_append_ms"] * 1e-3) / 1e9, 1),
            "smooth_search_append_ms": round(search["rope_smooth_append_ms"], 4),
            "smooth_search_append_GB/s": round(append_bytes / (search["rope_smooth_append_ms"] * 1e-3) / 1e9, 1)},
        "ffn_8192": {
            "what": "the FFN pair at 8192 tokens, outside the step: quantize A [8192x3072], up 3072->14336 with GELU "
                    "and the NVFP4 requant of its output (output scale from a calibration pass), down 14336->3072 to "
                    "bf16 on that NVFP4 output; each 2*M*N*K = 721.6 GFLOP",
            "quantize_ms": round(ffn["quantize_ms"], 4),
            "up_ms": round(ffn["up_ms"], 4),
            "up_TFLOP/s": round(2 * syn.FFN_UP.M * syn.FFN_UP.N * syn.FFN_UP.K / (ffn["up_ms"] * 1e-3) / 1e12, 1),
            "up_frac_fp4_peak": round(2 * syn.FFN_UP.M * syn.FFN_UP.N * syn.FFN_UP.K / (ffn["up_ms"] * 1e-3) / 1e12
                                      / fp4_peak, 4),
            "down_ms": round(ffn["down_ms"], 4),
            "down_TFLOP/s": round(2 * syn.FFN_DOWN.M * syn.FFN_DOWN.N * syn.FFN_DOWN.K / (ffn["down_ms"] * 1e-3)
                                  / 1e12, 1),
            "down_frac_fp4_peak": round(2 * syn.FFN_DOWN.M * syn.FFN_DOWN.N * syn.FFN_DOWN.K
                                        / (ffn["down_ms"] * 1e-3) / 1e12 / fp4_peak, 4)},
        "training": {
            "what": "training-side NVFP4 on the QKV layer shapes, outside the step: 2D (16x16) scaling of W "
                    "[9216x3072] writing W and W^T operands; RHT + transposed 1D quantize of X [4096x3072] and "
                    "dY [4096x9216] (weight-gradient operands); dW = dY^T X (9216x3072x4096) on those operands",
            "quantize_2d_ms": round(train["quantize_2d_ms"], 4),
            "quantize_2d_GB/s": round(N * K * 3.125 / (train["quantize_2d_ms"] * 1e-3) / 1e9, 1),
            "quantize_t_x_ms": round(train["quantize_t_x_ms"], 4),
            "quantize_t_x_GB/s": round(M * K * 2.5625 / (train["quantize_t_x_ms"] * 1e-3) / 1e9, 1),
            "quantize_t_dy_ms": round(train["quantize_t_dy_ms"], 4),
            "quantize_t_dy_GB/s": round(M * N * 2.5625 / (train["quantize_t_dy_ms"] * 1e-3) / 1e9, 1),
            "wgrad_ms": round(train["wgrad_ms"], 4),
            "wgrad_TFLOP/s": round(2.0 * N * K * M / (train["wgrad_ms"] * 1e-3) / 1e12, 1)},
        "kv_attention": {
            "what": "softmax attention of one 2640x24x128 bf16 query chunk over NVFP4 cache slots read directly "
                    "(e2m1 * s tiles in binary16, tcgen05 f16 MMAs with binary32 accumulators, one-pass softmax), "
                    "outside the step; TFLOP/s counts 4*Tq*keys*d*H",
            "bf16_peak_TFLOP/s": pk.get("bf16_tflops"), **attn},
        "ln_modulate_quantize": {
            "what": "LayerNorm + adaLN modulate + NVFP4 quantize of A, two launches, outside the step",
            "ms": round(search["ln_quantize_ms"], 4),
            "GB/s": round(quant_bytes / (search["ln_quantize_ms"] * 1e-3) / 1e9, 1)},
        "e2e": {"value": round(job_tflops(world, flops, e2e_ms), 3), "unit": "TFLOP/s",
                "h2d_bytes_per_step": M * K * 2, "d2h_bytes_per_step": M * N * 2,
                "what": "pinned host A -> device, quantize, gemm+bias, C -> pinned host, every step; the copies "
                        "run on their own streams (double-buffered) and overlap the neighbouring steps' compute"},
        "gpu_launches": 4 * args.steps,  # quantize, GEMM, KV append, KV dequant per step
        "clocks": clk,
    }
    return out


# --------------------------------------------------------------------------- oracle
def oracle_linear_rows(rows: int, w_codes, a_host, bias_host, seed_rows: int):
    """Time the CPU oracle on `rows` rows of the QKV layer: quantize those rows
    of A (with the full tensor scale), then their GEMM rows with bias."""
    import oracle

    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    sub = np.ascontiguousarray(a_host[:rows])
    t0 = time.perf_counter()
    codes, scales, a32 = oracle.quantize(sub)
    oracle.gemm((codes, scales, a32), w_codes, bias=bias_host, want_bf16=True)
    return time.perf_counter() - t0


def cpu_baseline(steps: int = 1, rows: int = 8) -> dict:
    import oracle

    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    a_host = syn.activations_bf16(M, K, seed=2)
    w_host = syn.normal_bf16((N, K), seed=3, std=0.02)
    bias_host = syn.normal_bf16((N,), seed=4, std=0.02)
    wq = oracle.quantize(w_host)
    ts = [oracle_linear_rows(rows, wq, a_host, bias_host, i) for i in range(steps)]
    t = min(ts)
    return {"value": round(2.0 * rows * N * K / t / 1e12, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(),
            "kind": "oracle", "host_cores": os.cpu_count(),
            "sample": f"{rows} of {M} token rows of the QKV layer per step (quantize rows + fp64 GEMM rows + bias)",
            "seconds_per_step": round(t, 3)}


def run_reference(args) -> dict:
    import oracle

    M, N, K = syn.QKV.M, syn.QKV.N, syn.QKV.K
    rows = 8
    a_host = syn.activations_bf16(M, K, seed=2)
    w_host = syn.normal_bf16((N, K), seed=3, std=0.02)
    bias_host = syn.normal_bf16((N,), seed=4, std=0.02)
    wq = oracle.quantize(w_host)
    for i in range(args.warmup):
        oracle_linear_rows(rows, wq, a_host, bias_host, i)
    t = 0.0
    for i in range(args.steps):
        t += oracle_linear_rows(rows, wq, a_host, bias_host, i)
    value = args.steps * 2.0 * rows * N * K / t / 1e12
    cb = {"value": round(value, 6), "unit": "TFLOP/s", "cores": oracle.get_threads(), "kind": "oracle",
          "sample": f"{rows} of {M} token rows of the QKV layer per step (quantize rows + fp64 GEMM rows + bias)"}
    return {"metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": round(1e3 * t / args.steps, 3), "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64 GEMM over NVFP4 operands; f32 quantize",
            "data": "synthetic (seeded, same generators as the GPU arm)", "impl": "reference",
            "config": {"workload": WORKLOAD, "M": M, "N": N, "K": K, "parallelism": "cpu oracle, rank 0"},
            "cpu_baseline": cb,
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
    if world > 1:
        import datetime

        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local))
    try:
        out = run_ours(args, rank, world)
        if rank == 0 and out is not None:
            if not args.no_cpu_baseline and world == 1:
                out["cpu_baseline"] = cpu_baseline()
            print(json.dumps(out), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
