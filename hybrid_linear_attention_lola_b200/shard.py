"""Sharding one batch's (batch, kv-head) streams over GPUs.

Every (batch, kv-head) stream of a LoLA layer is independent of the others: its
window, sparse cache and linear-attention state are its own, and the query heads
of a group read only their kv-head's stream. A batch therefore partitions over
ranks with no exchange on the data path: rank r owns a contiguous block of
sequences (when the world size divides the batch) or of kv-heads with their
query heads (when it divides the kv-heads), runs the engine on that shard, and
the outputs are gathered only where a caller wants them in one place.

This module holds the partition, the slicing of inputs into a shard and the
gather of the shard outputs (torch.distributed). The compute on a shard is a
callable, normally `LolaState.prefill` on this rank's GPU.
"""
from __future__ import annotations

import dataclasses
from typing import Callable, Optional


@dataclasses.dataclass(frozen=True)
class Shard:
    """Streams of one rank: sequences [b0, b1) x kv-heads [h0, h1) (query heads
    [h0 * g, h1 * g))."""
    rank: int
    world: int
    by: str            # "batch" or "kv_heads"
    b0: int
    b1: int
    h0: int
    h1: int
    g: int

    @property
    def batch(self) -> int:
        return self.b1 - self.b0

    @property
    def n_kv_heads(self) -> int:
        return self.h1 - self.h0

    @property
    def n_q_heads(self) -> int:
        return (self.h1 - self.h0) * self.g


def partition(batch: int, n_q_heads: int, n_kv_heads: int, world: int, rank: int) -> Shard:
    """Contiguous blocks of sequences when world divides batch, else of kv-heads when
    world divides n_kv_heads; every rank gets the same number of streams."""
    if world < 1 or not 0 <= rank < world:
        raise ValueError("rank outside the world")
    if n_q_heads % n_kv_heads:
        raise ValueError("n_q_heads must be a multiple of n_kv_heads")
    g = n_q_heads // n_kv_heads
    if batch % world == 0:
        per = batch // world
        return Shard(rank, world, "batch", rank * per, (rank + 1) * per, 0, n_kv_heads, g)
    if n_kv_heads % world == 0:
        per = n_kv_heads // world
        return Shard(rank, world, "kv_heads", 0, batch, rank * per, (rank + 1) * per, g)
    raise ValueError(f"{world} ranks divide neither the batch ({batch}) nor the kv-heads ({n_kv_heads})")


def shard_config(cfg, sh: Shard):
    """The engine config of one shard (a copy of cfg with the shard's sizes)."""
    import copy
    c = copy.copy(cfg)
    c.batch = sh.batch
    c.n_kv_heads = sh.n_kv_heads
    c.n_q_heads = sh.n_q_heads
    return c


def slice_inputs(sh: Shard, q, k, v):
    """The shard's q [b, t, hq, d] and k, v [b, t, hkv, d] (token-major, contiguous)."""
    qs = q[sh.b0:sh.b1, :, sh.h0 * sh.g:sh.h1 * sh.g]
    ks = k[sh.b0:sh.b1, :, sh.h0:sh.h1]
    vs = v[sh.b0:sh.b1, :, sh.h0:sh.h1]
    return qs.contiguous(), ks.contiguous(), vs.contiguous()


def slice_W(sh: Shard, W, per_kv_head: bool):
    """The shard's feature-map matrices: all of W when shared, its kv-heads' otherwise."""
    return W[sh.h0:sh.h1].contiguous() if per_kv_head else W


def gather(sh: Shard, out_local, group=None):
    """All-gathers the shard outputs [b, t, hq, d] into the full [B, t, Hq, d] on every
    rank (collective: every rank calls it in the same order)."""
    import torch
    import torch.distributed as dist
    parts = [torch.empty_like(out_local) for _ in range(sh.world)]
    dist.all_gather(parts, out_local.contiguous(), group=group)
    return torch.cat(parts, dim=0 if sh.by == "batch" else 2)


def run_sharded(sh: Shard, q, k, v, compute: Callable, group=None, gather_out: bool = True):
    """Slices this rank's streams out of q, k, v, runs `compute(q, k, v)` on them and
    (optionally) gathers every rank's outputs. Returns the local or full output."""
    out = compute(*slice_inputs(sh, q, k, v))
    return gather(sh, out, group) if gather_out else out
