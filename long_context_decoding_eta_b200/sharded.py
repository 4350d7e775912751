"""Sequence-sharded ETA decode over several GPUs (one process per GPU).

Every rank holds a block-aligned slice [t0, t1) of every row's KV cache
(`shard_range`), screens and decodes its slice with the ordinary step
(`EtaDecoder`, thresholds computed identically on every rank from the same
query), and the ranks' (o, lse) are gathered and merged with the log-sum-exp
identity (`eta_lse_merge`).  Screening is per block and the threshold per query,
so each shard admits exactly the blocks of the whole cache's union that fall in
its range, and the merge gives the decode of the whole cache (up to fp32
rounding of the merge).  The one exchange is the all-gather of B * Hq * (d + 1)
floats per rank (torch.distributed, NCCL between GPUs).

This module only allocates and calls: the step and the merge run in libeta.so.
"""
from __future__ import annotations

from typing import Optional, Tuple

import torch
import torch.distributed as dist

from . import _lib as L
from .api import EtaDecoder


def shard_range(T_max: int, blk: int, world: int, rank: int) -> Tuple[int, int]:
    """Token range [t0, t1) of rank `rank`: the cache's NB = T_max / blk blocks split
    into `world` contiguous runs of ceil(NB / world) blocks (the last runs may be
    shorter or empty)."""
    if T_max % blk or world <= 0 or not 0 <= rank < world:
        raise ValueError("T_max must be a multiple of blk and 0 <= rank < world")
    nb = T_max // blk
    per = -(-nb // world)
    b0 = min(rank * per, nb)
    b1 = min(b0 + per, nb)
    return b0 * blk, b1 * blk


def shard_lengths(lengths: torch.Tensor, t0: int, t1: int) -> torch.Tensor:
    """Valid keys of each row inside [t0, t1)."""
    return (lengths.to(torch.int64) - t0).clamp(0, t1 - t0).to(torch.int32)


def gather_parts(o: torch.Tensor, lse: torch.Tensor, group=None):
    """All-gather of every rank's (o, lse): returns o_parts [world, *o.shape] and
    lse_parts [world, *lse.shape] in rank order (identity without a process group)."""
    if not (dist.is_available() and dist.is_initialized()):
        return o.unsqueeze(0), lse.unsqueeze(0)
    world = dist.get_world_size(group)
    o_parts = torch.empty((world,) + tuple(o.shape), dtype=o.dtype, device=o.device)
    lse_parts = torch.empty((world,) + tuple(lse.shape), dtype=lse.dtype, device=lse.device)
    dist.all_gather(list(o_parts.unbind(0)), o.contiguous(), group=group)
    dist.all_gather(list(lse_parts.unbind(0)), lse.contiguous(), group=group)
    return o_parts, lse_parts


class ShardedEtaDecoder:
    """This rank's part of a sequence-sharded cache.

    K_shard, V_shard: bf16 [B, Hkv, t1 - t0, d] holding tokens [t0, t1) of every row
    (t1 - t0 a multiple of blk); lengths: int32 [B] of the whole cache.  Other
    arguments as EtaDecoder.  step() returns the merged (o, lse) of the whole cache on
    every rank."""

    def __init__(self, K_shard: torch.Tensor, V_shard: torch.Tensor, lengths: torch.Tensor,
                 t0: int, Hq: int, blk: int, group=None, **kw):
        self.t0, self.t1 = int(t0), int(t0) + int(K_shard.shape[2])
        self.group = group
        self.lengths = lengths
        self.dec = EtaDecoder(K_shard, V_shard, shard_lengths(lengths, self.t0, self.t1)
                              .to(K_shard.device), Hq, blk, **kw)
        self.o = torch.empty_like(self.dec.o)
        self.lse = torch.empty_like(self.dec.lse)

    def set_lengths(self, lengths: torch.Tensor):
        """New whole-cache lengths (after appending): this shard's share of them."""
        self.lengths = lengths
        self.dec.lengths.copy_(shard_lengths(lengths, self.t0, self.t1))

    def build_meta(self):
        self.dec.build_meta()

    def step(self, q, W=None, bias=None, tau_const=None, append: bool = True,
             stream: Optional[torch.cuda.Stream] = None):
        o, lse = self.dec.step(q, W, bias, tau_const, stream=stream, append=append)
        o_parts, lse_parts = gather_parts(o, lse, self.group)
        L.eta_lse_merge(o_parts, lse_parts, self.o, self.lse, stream)
        return self.o, self.lse
