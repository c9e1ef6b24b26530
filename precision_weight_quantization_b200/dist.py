"""NVFP4 on sibling groups whose tensors are sharded across data-parallel
ranks.

The global scale of an NVFP4 group is fl(A / 2688) with A the amax over every
element of every member (verl NVFP4 QAT article, 2.3 and 2.4: siblings share
one amax).  When a member is split across ranks, A is the one value the ranks
must exchange: each rank reduces its own shards (`nvfp4_group_amax`), one
all-reduce with MAX over a vector of all group amaxes makes them global, and
`nvfp4_quant` / `nvfp4_fake_quant` take it as `amax`.  Max is exact and does
not depend on the order of reduction, so every rank's codes, block scales and
global scales equal those of the unsharded call.  FP8 block and MXFP8 need no
exchange: their blocks never cross a shard boundary when shards are cut at
multiples of 128 rows (FP8 block) or anywhere along rows (MXFP8).
"""
from typing import List, Optional, Sequence

import torch
import torch.distributed as dist

from . import nvfp4_fake_quant, nvfp4_group_amax, nvfp4_quant


def allreduce_group_amax(amax: torch.Tensor, group=None) -> torch.Tensor:
    """All-reduce (MAX), in place, a 1-D FP32 vector of group amaxes (one per
    group and batch index).  A no-op without an initialised process group of
    more than one rank.  The tensor must live where the backend wants it
    (a CUDA tensor for NCCL, a CPU tensor for gloo)."""
    if amax.dtype != torch.float32 or amax.dim() != 1:
        raise ValueError("amax must be a 1-D float32 tensor")
    if dist.is_available() and dist.is_initialized() and dist.get_world_size(group) > 1:
        dist.all_reduce(amax, op=dist.ReduceOp.MAX, group=group)
    return amax


def sharded_group_amax(groups: Sequence[Sequence[torch.Tensor]], group=None) -> List[torch.Tensor]:
    """Global amax of every sibling group from this rank's shards.

    groups[g] lists this rank's shards of group g's members (BF16, on this
    rank's GPU, every group with the same batch count on every rank).
    Returns one FP32 tensor of shape [B_g] per group, identical on every
    rank.  One collective for all groups."""
    local = [nvfp4_group_amax(list(g)).reshape(-1) for g in groups]
    sizes = [t.numel() for t in local]
    vec = torch.cat(local) if local else torch.empty(0, dtype=torch.float32)
    allreduce_group_amax(vec, group)
    return list(torch.split(vec, sizes))


def nvfp4_quant_sharded(groups: Sequence[Sequence[torch.Tensor]], group=None):
    """NVFP4 quantisation of this rank's shards with each group's global
    amax.  Returns [(packed, block scales, global scale)] per group, as
    `nvfp4_quant`."""
    amax = sharded_group_amax(groups, group)
    return [nvfp4_quant(list(g), amax=a) for g, a in zip(groups, amax)]


def nvfp4_fake_quant_sharded(groups: Sequence[Sequence[torch.Tensor]], group=None,
                             inplace: bool = False) -> List:
    """NVFP4 fake-quantisation of this rank's shards with each group's global
    amax.  Returns the BF16 outputs per group, as `nvfp4_fake_quant`."""
    amax = sharded_group_amax(groups, group)
    return [nvfp4_fake_quant(list(g), amax=a, inplace=inplace) for g, a in zip(groups, amax)]


def row_shard(x: torch.Tensor, rank: int, world: int, multiple: int = 1) -> torch.Tensor:
    """Rows [r0, r1) of x for `rank` of `world`, cut at multiples of
    `multiple` rows (128 keeps FP8 tiles whole); a view, possibly empty."""
    M = x.shape[-2]
    units = -(-M // multiple)
    per = -(-units // world)
    r0 = min(M, rank * per * multiple)
    r1 = min(M, (rank + 1) * per * multiple)
    return x[..., r0:r1, :]
