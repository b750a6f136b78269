"""Token-sharded NVFP4 activations across ranks.

When the tokens of one activation are split across GPUs (each rank holds a
block of rows; the weights are replicated), every rank quantizes its own rows,
but the FP32 tensor scale of the NVFP4 format belongs to the whole tensor
("LongLive-2.0：用 NVFP4 并行底座做长视频生成", yingwang.github.io reading note,
二 方法 / "NVFP4 量化格式": one FP32 scale per tensor, one E4M3 scale per
16-element block).  The ranks therefore agree on it before their encode: each
computes its local scale a32_r = fl32(amax_r / 2688), and one 4-byte
all-reduce-max gives max_r a32_r.  Binary32 division by 2688 rounds
monotonically, so this max equals fl32(max_r amax_r / 2688): exactly the
scale of the unsplit tensor, and the ranks' codes concatenate to those of a
single-rank quantize.  Without the all-reduce each shard gets its own scale
(a per-shard tensor scale), which changes the codes of every shard that does
not hold the tensor's maximum.

This module only issues the collective; the quantize is the library's.
"""
from __future__ import annotations

import torch
import torch.distributed as dist


def shared_tensor_scale(local_a32: torch.Tensor, group=None) -> torch.Tensor:
    """The tensor scale of the whole token-sharded tensor: the maximum over the
    ranks of their local binary32 scales (a 1-element float32 tensor, on the
    device the group's backend uses).  Returns a new tensor."""
    t = local_a32.detach().reshape(1).to(torch.float32).clone()
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX, group=group)
    return t


def quantize_shard(x_local: torch.Tensor, group=None, *, ws=None, stream=None):
    """NVFP4 quantize of this rank's rows with the tensor scale of the whole
    token-sharded tensor: the local quantize computes a32_r, the ranks agree on
    the maximum, and the rows are encoded again with it when it differs from
    the local one (the rank holding the tensor's maximum keeps its first
    encode)."""
    from . import nvfp4 as nv

    q = nv.quantize(x_local, ws=ws, stream=stream)
    a = shared_tensor_scale(q.global_scale, group)
    if not torch.equal(a, q.global_scale):
        q = nv.quantize(x_local, global_scale=a, out=q, ws=ws, stream=stream)
    return q
