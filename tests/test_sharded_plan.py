"""Host-side plan of split-KV across GPUs (CPU only).

Every rank must own a contiguous run of each sequence's blocks, the runs of all
ranks must partition the sequence's blocks in order, and the local key counts
must add up to the context length: then the log-sum-exp combination of the
ranks' partials covers every key exactly once.  Checked in one process for
many shapes, and across two gloo ranks exchanging their plans.
"""
import os
import socket

import numpy as np
import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

from paged_kv_cache_331_b200.sharded import shard_block_range, shard_tables


def _check_partition(bt, lens, bs, world, plans):
    nbs = (lens + bs - 1) // bs
    for b in range(len(lens)):
        blocks = []
        for local, local_lens in plans:
            n = int((local[b] >= 0).sum())
            assert (local[b, :n] >= 0).all() and (local[b, n:] == -1).all()
            blocks.extend(local[b, :n].tolist())
        assert blocks == bt[b, :nbs[b]].tolist()
        assert sum(int(ll[b]) for _, ll in plans) == lens[b]


@pytest.mark.parametrize("world", [1, 2, 3, 8])
@pytest.mark.parametrize("bs", [16, 256])
def test_shards_partition_every_sequence(world, bs):
    rng = np.random.default_rng(world * 1000 + bs)
    lens = np.concatenate([[0, 1, bs - 1, bs, bs + 1, 3 * bs], rng.integers(0, 40 * bs, 20)]).astype(np.int32)
    nbs = (lens + bs - 1) // bs
    bt = np.full((len(lens), int(nbs.max())), -1, np.int32)
    perm = rng.permutation(int(nbs.sum()))
    o = 0
    for b, n in enumerate(nbs):
        bt[b, :n] = perm[o:o + n]
        o += n
    plans = [shard_tables(bt, lens, bs, world, r) for r in range(world)]
    _check_partition(bt, lens, bs, world, plans)
    for r in range(world):                                  # contiguous, balanced runs
        for n in nbs:
            lo, hi = shard_block_range(int(n), world, r)
            assert hi - lo in ((int(n) // world), (int(n) + world - 1) // world)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = np.random.default_rng(7)                      # every rank sees the same global plan
        bs = 16
        lens = rng.integers(0, 600, 9).astype(np.int32)
        nbs = (lens + bs - 1) // bs
        bt = np.full((9, int(nbs.max())), -1, np.int32)
        ids = rng.permutation(int(nbs.sum()))
        o = 0
        for b, n in enumerate(nbs):
            bt[b, :n] = ids[o:o + n]
            o += n
        mine = shard_tables(bt, lens, bs, world, rank)
        gathered = [None] * world
        dist.all_gather_object(gathered, mine)
        if rank == 0:
            _check_partition(bt, lens, bs, world, gathered)
        out.put(rank)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_exchange_a_partition():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(120)
        assert p.exitcode == 0
    assert sorted(q.get(timeout=10) for _ in range(2)) == [0, 1]


def _exchange_main(rank, world, port, out):
    """Each rank computes its partial over its shard with the oracle, in the library's format (fp32 o = acc / l,
    lse in log2 units), exchanges it through ShardedDecode.gather, and rank 0 checks the gathered layout
    [R, B, Hq, ...]: merged by the oracle's log-sum-exp merge (ranks as chunks) it must equal the oracle's
    unsplit decode."""
    import math
    import torch
    from oracle import oracle as O
    from paged_kv_cache_331_b200 import workloads as W
    from paged_kv_cache_331_b200.sharded import ShardedDecode
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        orc = O.get()
        w = W.decode_workload(np.array([700, 1, 33, 260], np.int32), 8, 2, 64, 16, rng=np.random.default_rng(11))
        lt, ll = shard_tables(w.block_tables, w.context_lens, w.block_size, world, rank)
        m, l, acc = orc.decode_partials(w.q, w.k_cache, w.v_cache, lt, ll, w.scale, max(int(ll.max()), 1), 1)
        empty = (ll == 0)[:, None]
        o = np.where(empty[..., None], 0.0, acc[:, :, 0, :] / np.where(empty, 1.0, l[:, :, 0])[..., None])
        lse = np.where(empty, -np.inf, (m[:, :, 0] + np.log(np.where(empty, 1.0, l[:, :, 0]))) / math.log(2.0))
        sd = ShardedDecode()
        o_all = sd.gather(torch.from_numpy(o.astype(np.float32)))
        lse_all = sd.gather(torch.from_numpy(lse.astype(np.float32)))
        assert tuple(o_all.shape) == (world,) + o.shape and tuple(lse_all.shape) == (world,) + lse.shape
        if rank == 0:
            mr = lse_all.double().numpy().transpose(1, 2, 0) * math.log(2.0)       # [B, Hq, R], natural units
            lr = np.ones_like(mr)
            ar = o_all.double().numpy().transpose(1, 2, 0, 3)                       # [B, Hq, R, D]
            _, merged = orc.merge_partials(mr, lr, ar)
            _, ref = orc.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
            np.testing.assert_allclose(merged, ref, rtol=0, atol=1e-6)            # fp32 partials
        out.put(rank)
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_gather_partials_in_the_merge_layout():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_exchange_main, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(180)
        assert p.exitcode == 0
    assert sorted(q.get(timeout=10) for _ in range(2)) == [0, 1]


def test_injected_gather_is_checked_for_its_layout():
    import torch
    from paged_kv_cache_331_b200.sharded import ShardedDecode
    good = ShardedDecode(gather=lambda t: torch.stack([t, t + 1]), world=2)
    g = good.gather(torch.zeros(3, 4))
    assert tuple(g.shape) == (2, 3, 4) and bool((g[1] == 1).all())
    bad = ShardedDecode(gather=lambda t: torch.cat([t, t]), world=2)      # concatenated, not stacked
    with pytest.raises(ValueError):
        bad.gather(torch.zeros(3, 4))
    with pytest.raises(ValueError):
        ShardedDecode(gather=lambda t: t)
