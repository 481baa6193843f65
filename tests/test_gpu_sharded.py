"""Split-KV across GPUs, with the ranks emulated one after another on one GPU.

Each emulated rank runs pa_decode_partial over its share of every sequence's
blocks (shard_tables); pa_merge_partials combines the stacked partials.  The
result must match the oracle's unsplit decode within the attention tolerance,
and every partial must match the oracle restricted to that rank's keys:
- o against the oracle's fp64 decode over the shard;
- lse against log2(e) * (m + ln l) of the oracle's one-chunk partial.

The ranks' kernels never wait on one another.  Each launch completes on its
own, so running them in sequence on one device is exact.
"""
import math

import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from paged_kv_cache_331_b200.sharded import shard_tables
from gpu_helpers import DeviceDecode, assert_attention_close, dev_i32

pytestmark = pytest.mark.gpu

CASES = [  # context lengths, Hq, Hkv, D, block size, ranks, kv_chunk_size
    ([5000, 1, 0, 300, 257], 32, 8, 128, 256, 3, 0),
    ([9000, 17], 16, 2, 128, 16, 8, 0),
    ([100, 2000, 65], 8, 8, 64, 64, 2, 64),
    ([40000, 3], 32, 8, 128, 256, 4, 0),
    ([700, 700, 700, 700], 4, 1, 64, 16, 1, 128),
]


@pytest.mark.parametrize("lens,hq,hkv,d,bs,world,chunk", CASES)
def test_sharded_partials_merge_to_the_unsplit_decode(oracle, lens, hq, hkv, d, bs, world, chunk):
    rng = np.random.default_rng(sum(lens) + world)
    w = W.decode_workload(np.array(lens, np.int32), hq, hkv, d, bs, rng=rng)
    dw = DeviceDecode(w)
    parts_o, parts_lse = [], []
    for r in range(world):
        lt, ll = shard_tables(w.block_tables, w.context_lens, bs, world, r)
        o, lse = pa.decode_partial(dw.q, dw.k_cache, dw.v_cache, dev_i32(lt), dev_i32(ll), int(ll.max()), w.scale,
                                   kv_chunk_size=chunk)
        torch.cuda.synchronize()
        og, lg = o.cpu().numpy(), lse.cpu().numpy()
        # this rank's partial against the oracle over the same keys
        _, o_ref = oracle.decode(w.q, w.k_cache, w.v_cache, lt, ll, w.scale, want_f64=True)
        m, l, _ = oracle.decode_partials(w.q, w.k_cache, w.v_cache, lt, ll, w.scale, max(int(ll.max()), 1), 1)
        empty = ll == 0
        assert (og[empty] == 0).all() and np.isneginf(lg[empty]).all()
        live = ~empty
        if live.any():
            np.testing.assert_allclose(og[live], o_ref[live], rtol=0, atol=5e-4)
            lse_ref = (m[live, :, 0] + np.log(l[live, :, 0])) / math.log(2.0)
            np.testing.assert_allclose(lg[live], lse_ref, rtol=0, atol=2e-3)
        parts_o.append(o)
        parts_lse.append(lse)
    out = pa.merge_partials(torch.stack(parts_o), torch.stack(parts_lse))
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    torch.cuda.synchronize()
    assert_attention_close(out, ref, what=f"sharded decode over {world} ranks")
    # one rank holding everything is plain decode
    if world == 1:
        full = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, int(max(lens)), w.scale,
                         kv_chunk_size=chunk)
        assert (full.float() - out.float()).abs().max().item() <= 2 ** -7
    assert pa.device_error() == 0


def test_merge_partials_matches_the_oracle_merge(oracle):
    """pa_merge_partials on random partials against the oracle's log-sum-exp merge."""
    rng = np.random.default_rng(11)
    R, B, H, D = 5, 3, 4, 128
    o = rng.standard_normal((R, B, H, D)).astype(np.float32)
    lse = (rng.standard_normal((R, B, H)) * 20).astype(np.float32)
    lse[1, 0, :] = -np.inf                        # a rank without keys for sequence 0
    lse[:, 2, 3] = -np.inf                        # a row with no keys anywhere
    out = pa.merge_partials(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda())
    torch.cuda.synchronize()
    # the oracle's merge takes (m, l, acc) per chunk: m = lse * ln 2, l = 1, acc = o
    m = np.moveaxis(lse.astype(np.float64) * math.log(2.0), 0, -1)
    l = np.where(np.isneginf(m), 0.0, 1.0)
    acc = np.moveaxis(o.astype(np.float64), 0, 2) * l[..., None]
    ref_bits, ref = oracle.merge_partials(m, l, acc)
    got = out.float().cpu().numpy()
    assert np.abs(got - ref).max() <= 2 ** -7 * max(1.0, np.abs(ref).max())
    assert (got[2, 3] == 0).all()


def test_sharded_decode_call_with_an_injected_gather(oracle):
    """ShardedDecode.__call__ (partial, exchange, merge) for every emulated rank of 3: the exchange is a gather that
    puts this rank's partial at its index among the other ranks' partials, computed beforehand, as the all-gather
    would.  Every rank's output must be the same and match the oracle's unsplit decode."""
    from paged_kv_cache_331_b200.sharded import ShardedDecode
    lens, hq, hkv, d, bs, world = [5000, 1, 300, 257], 32, 8, 128, 256, 3
    rng = np.random.default_rng(91)
    w = W.decode_workload(np.array(lens, np.int32), hq, hkv, d, bs, rng=rng)
    dw = DeviceDecode(w)
    plans = [shard_tables(w.block_tables, w.context_lens, bs, world, r) for r in range(world)]
    parts = [pa.decode_partial(dw.q, dw.k_cache, dw.v_cache, dev_i32(lt), dev_i32(ll), int(ll.max()), w.scale)
             for lt, ll in plans]
    outs = []
    for r, (lt, ll) in enumerate(plans):
        def gather(t, r=r):
            others = [p[0] if t.dim() == 3 else p[1] for p in parts]
            return torch.stack([t if i == r else others[i] for i in range(world)])
        sd = ShardedDecode(gather=gather, world=world)
        outs.append(sd(dw.q, dw.k_cache, dw.v_cache, dev_i32(lt), dev_i32(ll), int(ll.max()), w.scale))
    torch.cuda.synchronize()
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(outs[0], ref, what="ShardedDecode over 3 emulated ranks")
    assert pa.device_error() == 0
