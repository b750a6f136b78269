"""Token-sharded quantize on two gloo ranks (CPU): the QKV activation's tokens
split in two, each rank quantizing its rows with the oracle standing in for the
library's quantize.  With the 4-byte all-reduce-max of the tensor scale
(bit_video_dit_b200.shard.shared_tensor_scale) the ranks' codes and scales
concatenate to the single-rank quantize bit for bit; without it, each shard's
scale is its own: equal to the whole tensor's on the rank holding the maximum
(whose rows then match), smaller on the other (whose rows do not)."""
import os
import socket

import numpy as np
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from bit_video_dit_b200 import synthetic as syn
from bit_video_dit_b200.shard import shared_tensor_scale

ROWS, COLS = 512, syn.QKV.K


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, q):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        x = syn.activations_bf16(ROWS, COLS, seed=2)
        n = ROWS // world
        mine = np.ascontiguousarray(x[rank * n:(rank + 1) * n])
        c_local, s_local, a_local = oracle.quantize(mine)
        a_shared = shared_tensor_scale(torch.tensor([a_local], dtype=torch.float32))
        a = np.float32(a_shared.item())
        c, s, _ = oracle.quantize(mine, a)
        q.put((rank, a_local, a, c, s, c_local, s_local))
    finally:
        dist.destroy_process_group()


def test_shared_tensor_scale_reproduces_the_single_rank_quantize():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r = q.get(timeout=300)
        res[r[0]] = r[1:]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    x = syn.activations_bf16(ROWS, COLS, seed=2)
    c_ref, s_ref, a_ref = oracle.quantize(x)
    bits = lambda v: int(np.float32(v).view(np.uint32))
    # shared scale: every rank has the whole tensor's scale, and the shards concatenate exactly
    for r in range(world):
        assert bits(res[r][1]) == bits(a_ref)
    assert np.array_equal(np.concatenate([res[r][2] for r in range(world)]), c_ref)
    assert np.array_equal(np.concatenate([res[r][3] for r in range(world)]), s_ref)
    # per-shard scales: the rank holding the maximum has the tensor's scale and its rows match;
    # the other rank's scale is smaller and its codes differ
    n = ROWS // world
    top = max(range(world), key=lambda r: res[r][0])
    assert bits(res[top][0]) == bits(a_ref)
    assert np.array_equal(res[top][4], c_ref[top * n:(top + 1) * n])
    for r in range(world):
        if r != top:
            assert res[r][0] < a_ref
            assert not np.array_equal(res[r][4], c_ref[r * n:(r + 1) * n])


def test_single_process_leaves_the_scale_alone():
    t = torch.tensor([0.125], dtype=torch.float32)
    assert torch.equal(shared_tensor_scale(t), t)
