"""Batch sharding of the PRR decode step over GPUs (one process per GPU, or one
process driving several GPUs).

Every (sequence, KV head) unit is independent in every step of the method -- block
scoring, top-K, speculation, repair, merge and the EMA predictor -- so a batch splits
across devices with no exchange on the data path: each device holds the caches,
summaries and predictor state of its own sequences and runs the whole step on them.
Sequences are the sharding grain (a sequence's KV heads share its query and length).

Only a caller that wants every sequence's output on one rank needs a collective, and
that is outside the step: gather_outputs concatenates the shards' [out | lse] rows in
sequence order with one all-gather over whatever torch.distributed group it is given.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, List, Optional, Sequence, Tuple

import torch

from ._abi import Dims


def shard_ranges(B: int, world: int) -> List[Tuple[int, int]]:
    """Contiguous sequence ranges [b0, b1) of each shard: sizes differ by at most one,
    the larger shards first; a shard may be empty when world > B."""
    if B < 0 or world < 1:
        raise ValueError("need B >= 0 and world >= 1")
    base, extra = divmod(B, world)
    out, b0 = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        out.append((b0, b0 + n))
        b0 += n
    return out


def shard_dims(dims: Dims, rng: Tuple[int, int]) -> Dims:
    """Dims of one shard: the same shape with the shard's batch."""
    return dataclasses.replace(dims, B=rng[1] - rng[0])


def gather_outputs(local: torch.Tensor, ranges: Sequence[Tuple[int, int]], group=None) -> torch.Tensor:
    """All-gather the shards' per-sequence rows (local: [b1-b0][...] of this rank) into
    [B][...] in sequence order.  Shards of unequal size are padded for the collective
    and trimmed after it.  Every rank of the group calls it with its own rows."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    if len(ranges) != world:
        raise ValueError("one range per rank")
    rows = max(b1 - b0 for b0, b1 in ranges)
    pad = torch.zeros((rows,) + tuple(local.shape[1:]), dtype=local.dtype, device=local.device)
    pad[:local.shape[0]] = local
    parts = [torch.empty_like(pad) for _ in range(world)]
    dist.all_gather(parts, pad, group=group)
    return torch.cat([parts[r][:b1 - b0] for r, (b0, b1) in enumerate(ranges)], dim=0)


class ShardedDecoder:
    """A batch of sequences decoded by several independent PRRDecoders.

    `devices`: the CUDA devices of this process.  Under one process per GPU (torchrun),
    pass this rank's device and `rank`/`world` -- the process then owns only its shard.
    In one process with several GPUs, pass all devices and world = len(devices).  The
    step is launched on every local shard without any synchronisation between them."""

    def __init__(self, dims: Dims, devices: Sequence[torch.device], rank: int = 0, world: Optional[int] = None,
                 make: Optional[Callable[[Dims, torch.device], object]] = None):
        from .decoder import PRRDecoder
        world = len(devices) if world is None else world
        self.dims = dims
        self.ranges = shard_ranges(dims.B, world)
        local = list(range(world)) if len(devices) == world else [rank]
        if len(devices) != len(local):
            raise ValueError("pass one device per local shard")
        build = make or (lambda d, dev: PRRDecoder(d, device=dev))
        self.shards = [(self.ranges[r], build(shard_dims(dims, self.ranges[r]), devices[i]))
                       for i, r in enumerate(local) if self.ranges[r][1] > self.ranges[r][0]]

    def step_fused(self, q: torch.Tensor, k_new: torch.Tensor, v_new: torch.Tensor) -> None:
        """One decode step on every local shard: q [B][Hq][d], k_new / v_new [B][Hkv][d]
        bf16 (full batch, any device); each shard copies its own sequences' rows on its
        step stream (after the caller's current stream) and appends its token inside
        its fused launch."""
        for (b0, b1), dec in self.shards:
            with torch.cuda.device(dec.device):
                dec.step_fused(q[b0:b1], k_new=k_new[b0:b1], v_new=v_new[b0:b1])

    def outputs(self) -> List[Tuple[Tuple[int, int], torch.Tensor, torch.Tensor]]:
        """(sequence range, out, lse) of every local shard, on its own device."""
        return [(rng, dec.out, dec.lse) for rng, dec in self.shards]

    def synchronize(self) -> None:
        for _, dec in self.shards:
            dec.select_stream.synchronize()
