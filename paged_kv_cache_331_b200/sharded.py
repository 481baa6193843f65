"""Decode for sequences whose KV cache is spread over several GPUs (split-KV
across devices).

Each rank holds a contiguous run of every sequence's cache blocks (rank r owns
logical blocks [floor(nb*r/W), floor(nb*(r+1)/W)) of a sequence with nb
blocks).  A decode step then is:

    pa_decode_partial   on every rank, over its own blocks: fp32 (o, lse)
    all-gather          of the partials (NCCL over NVLink / NVSwitch)
    pa_merge_partials   on every rank: the log-sum-exp combination

The combination is the in-GPU split-KV merge of pa_decode applied across
devices, so the result equals single-GPU decode up to rounding.  Only the
partials cross NVLink (Hq * (D + 1) * 4 bytes per sequence and rank), never
the cache.  The pages' engine shards attention by heads, which needs no
exchange inside attention ("Architektur im Überblick",
Tensor-Parallelität); this module covers contexts too long for one GPU's
cache.
"""
from __future__ import annotations

import numpy as np
import torch

from . import _binding as pa


def shard_block_range(num_blocks: int, world: int, rank: int):
    """Logical blocks [lo, hi) of a sequence with num_blocks blocks that rank owns."""
    return (num_blocks * rank) // world, (num_blocks * (rank + 1)) // world


def shard_tables(block_tables: np.ndarray, context_lens: np.ndarray, block_size: int, world: int, rank: int):
    """Split host-side block tables by rank.

    Returns (local_tables [B, width], local_lens [B]): rank's blocks of each
    sequence, left-aligned and padded with -1, and the number of keys they
    hold.
    """
    if not 0 <= rank < world:
        raise ValueError("rank out of range")
    bt = np.asarray(block_tables, dtype=np.int32)
    lens = np.asarray(context_lens, dtype=np.int64)
    B = bt.shape[0]
    nbs = (lens + block_size - 1) // block_size
    width = max(1, int(max(((n * (rank + 1)) // world - (n * rank) // world) for n in nbs)) if B else 1)
    local = np.full((B, width), -1, np.int32)
    local_lens = np.zeros(B, np.int32)
    for b in range(B):
        lo, hi = shard_block_range(int(nbs[b]), world, rank)
        local[b, :hi - lo] = bt[b, lo:hi]
        local_lens[b] = max(0, min(hi * block_size, int(lens[b])) - lo * block_size) if hi > lo else 0
    return local, local_lens


class ShardedDecode:
    """One decode step over a context sharded across the ranks of a process group.

    ``gather(t)`` returns the ranks' copies of ``t`` stacked along a new leading
    axis, ``[world, *t.shape]``, rank r's at index r.  By default it is an
    all-gather over ``group`` (NCCL over NVLink for CUDA tensors, gloo for CPU
    tensors); a caller may pass its own exchange with the same contract
    (``world`` is then required).
    """

    def __init__(self, group=None, *, gather=None, world=None):
        if gather is None:
            import torch.distributed as dist
            self.dist = dist
            self.group = group
            self.world = dist.get_world_size(group)
            self._gather = self._all_gather
        else:
            if world is None or world < 1:
                raise ValueError("an injected gather needs the world size")
            self.dist, self.group, self.world = None, group, int(world)
            self._gather = gather

    def _all_gather(self, t):
        t = t.contiguous()
        # concatenated along dim 0 (the layout both NCCL and gloo accept), then viewed as [world, *shape]
        out = torch.empty((self.world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
        self.dist.all_gather_into_tensor(out, t, group=self.group)
        return out.view((self.world,) + tuple(t.shape))

    def gather(self, t):
        g = self._gather(t)
        if tuple(g.shape) != (self.world,) + tuple(t.shape):
            raise ValueError(f"gather returned shape {tuple(g.shape)}, expected {(self.world,) + tuple(t.shape)}")
        return g

    def __call__(self, q, k_cache, v_cache, local_tables, local_lens, max_local_len, scale, *, out=None,
                 kv_chunk_size=0):
        """pa_decode_partial over this rank's blocks, the all-gather of (o, lse), then pa_merge_partials."""
        o, lse = pa.decode_partial(q, k_cache, v_cache, local_tables, local_lens, max_local_len, scale,
                                   kv_chunk_size=kv_chunk_size)
        return pa.merge_partials(self.gather(o), self.gather(lse), out=out)
