"""CUDA-graph capture of the store + decode step (captured at the batch sizes
of "Architektur im Überblick", CUDA Graph Optimierung), against eager calls
and the oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from paged_kv_cache_331_b200.graphs import DecodeGraphRunner
from gpu_helpers import DeviceDecode, assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("n", [20, 1, 5, 16, 32])
def test_graph_replay_matches_eager_and_oracle(oracle, n):
    rng = np.random.default_rng(100 + n)
    lens = rng.integers(1, 1500, size=n).astype(np.int32)
    w = W.decode_workload(lens, 8, 2, 128, 256, rng=rng)
    dw = DeviceDecode(w)
    chunk = 256
    runner = DecodeGraphRunner(dw.k_cache, dw.v_cache, w.num_heads, max_bs=32, max_blocks_per_seq=8,
                               max_context_len=2048, scale=w.scale, kv_chunk_size=chunk)
    # the graph path stores the new rows itself; the eager reference works on its own copy of the cache
    kc2, vc2 = dw.k_cache.clone(), dw.v_cache.clone()
    out_g = runner.run(dw.q, dw.new_k, dw.new_v, dw.slot_mapping, dw.block_tables, dw.context_lens).clone()
    pa.store_kvcache(dw.new_k, dw.new_v, kc2, vc2, dw.slot_mapping)
    out_e = pa.decode(dw.q, kc2, vc2, dw.block_tables, dw.context_lens, 2048, w.scale, kv_chunk_size=chunk)
    torch.cuda.synchronize()
    assert torch.equal(dw.k_cache.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16))
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out_g, ref, what=f"graph replay n={n}")
    # a second replay of the same step is bitwise identical
    out_g2 = runner.run(dw.q, dw.new_k, dw.new_v, dw.slot_mapping, dw.block_tables, dw.context_lens)
    torch.cuda.synchronize()
    assert torch.equal(out_g.view(torch.int16), out_g2.view(torch.int16))
    assert pa.device_error() == 0


@pytest.mark.parametrize("n", [3, 16])
def test_rotary_graph_replay_matches_eager_and_oracle(oracle, n):
    rng = np.random.default_rng(200 + n)
    lens = rng.integers(1, 2000, size=n).astype(np.int32)
    w = W.decode_workload(lens, 16, 8, 128, 256, rng=rng)
    dw = DeviceDecode(w)
    table = oracle.rope_table(2048, 128, 1e6)
    dtab = torch.from_numpy(table).cuda()
    pos = torch.from_numpy(lens - 1).cuda()
    runner = DecodeGraphRunner(dw.k_cache, dw.v_cache, w.num_heads, max_bs=16, max_blocks_per_seq=8,
                               max_context_len=2048, scale=w.scale, cos_sin_cache=dtab)
    kc2, vc2 = dw.k_cache.clone(), dw.v_cache.clone()
    out_g = runner.run(dw.q, dw.new_k, dw.new_v, dw.slot_mapping, dw.block_tables, dw.context_lens, pos).clone()
    qr = pa.rotary_store_kvcache(dw.q, dw.new_k, dw.new_v, pos, dtab, kc2, vc2, dw.slot_mapping)
    out_e = pa.decode(qr, kc2, vc2, dw.block_tables, dw.context_lens, 2048, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(dw.k_cache.view(torch.int16), kc2.view(torch.int16))
    assert torch.equal(out_g.view(torch.int16), out_e.view(torch.int16))
    q_rot = oracle.rope_store_kvcache(w.q, w.new_k, w.new_v, lens - 1, table, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(q_rot, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out_g, ref, what=f"rotary graph replay n={n}")
    assert pa.device_error() == 0


def test_host_decode_step_matches_the_device_calls(oracle):
    from paged_kv_cache_331_b200.graphs import HostDecodeStep
    rng = np.random.default_rng(77)
    lens = rng.integers(1, 3000, 12).astype(np.int32)
    w = W.decode_workload(lens, 16, 8, 128, 256, rng=rng)
    a, b = DeviceDecode(w), DeviceDecode(w)
    step = HostDecodeStep(a.k_cache, a.v_cache, 12, 16, w.block_tables.shape[1], 3072, w.scale)
    h = step.inputs()
    for name, arr in (("q", w.q), ("new_k", w.new_k), ("new_v", w.new_v)):
        h[name].view(torch.int16).copy_(torch.from_numpy(arr.view(np.int16)))
    h["slot_mapping"].copy_(torch.from_numpy(w.slot_mapping))
    h["block_tables"].copy_(torch.from_numpy(w.block_tables))
    h["context_lens"].copy_(torch.from_numpy(w.context_lens))
    out_h = step.run().clone()
    ref = pa.store_decode(b.q, b.new_k, b.new_v, b.slot_mapping, b.k_cache, b.v_cache, b.block_tables,
                          b.context_lens, 3072, w.scale)
    torch.cuda.synchronize()
    assert torch.equal(out_h.view(torch.int16), ref.cpu().view(torch.int16))
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert torch.equal(step.run().view(torch.int16), out_h.view(torch.int16))   # a second replay
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, f64 = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out_h, f64, what="host decode step")
    assert pa.device_error() == 0


def test_host_decode_pipeline_overlapped_steps_match_sequential_calls(oracle):
    """Five generation steps through the double-buffered host pipeline: every step appends one token to each
    sequence (its own q and new K/V row, context one longer), the next step is submitted before the previous
    one is waited for, and each step's host output must equal the same steps run one by one with
    pa_store_decode (bitwise) and the oracle's store + decode chain (within tolerance)."""
    from paged_kv_cache_331_b200.graphs import HostDecodePipeline
    rng = np.random.default_rng(78)
    steps = 5
    final = rng.integers(steps + 1, 3000, 12).astype(np.int32)
    w = W.decode_workload(final, 16, 8, 128, 256, rng=rng)
    B = w.num_seqs
    qs = [W.randn_bf16(rng, w.q.shape) for _ in range(steps)]
    nks = [W.randn_bf16(rng, w.new_k.shape) for _ in range(steps)]
    nvs = [W.randn_bf16(rng, w.new_v.shape) for _ in range(steps)]
    lens = [final - (steps - 1) + k for k in range(steps)]
    slots = [np.array([W.slots_for_positions(w.block_tables[b], [int(lens[k][b]) - 1], 256)[0] for b in range(B)],
                      np.int32) for k in range(steps)]
    a, b = DeviceDecode(w), DeviceDecode(w)
    pipe = HostDecodePipeline(a.k_cache, a.v_cache, B, 16, w.block_tables.shape[1], 3072, w.scale)
    bf = lambda arr: torch.from_numpy(np.ascontiguousarray(arr).view(np.int16))   # noqa: E731
    outs, tickets = [], []
    for k in range(steps):
        if k >= pipe.depth:                           # the slot's previous step must have come back
            outs.append(pipe.wait(tickets[k - pipe.depth]).clone())
        h = pipe.inputs(pipe.next_slot())
        h["q"].view(torch.int16).copy_(bf(qs[k]))
        h["new_k"].view(torch.int16).copy_(bf(nks[k]))
        h["new_v"].view(torch.int16).copy_(bf(nvs[k]))
        h["slot_mapping"].copy_(torch.from_numpy(slots[k]))
        h["block_tables"].copy_(torch.from_numpy(w.block_tables))
        h["context_lens"].copy_(torch.from_numpy(lens[k]))
        tickets.append(pipe.submit())
    for t in tickets[len(outs):]:
        outs.append(pipe.wait(t).clone())
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    for k in range(steps):
        dq = torch.from_numpy(qs[k].view(np.int16)).view(torch.bfloat16).cuda()
        dk = torch.from_numpy(nks[k].view(np.int16)).view(torch.bfloat16).cuda()
        dv = torch.from_numpy(nvs[k].view(np.int16)).view(torch.bfloat16).cuda()
        ref = pa.store_decode(dq, dk, dv, torch.from_numpy(slots[k]).cuda(), b.k_cache, b.v_cache, b.block_tables,
                              torch.from_numpy(lens[k]).cuda(), 3072, w.scale)
        torch.cuda.synchronize()
        assert torch.equal(outs[k].view(torch.int16), ref.cpu().view(torch.int16)), f"step {k}"
        oracle.store_kvcache(nks[k], nvs[k], kc, vc, slots[k])
        _, f64 = oracle.decode(qs[k], kc, vc, w.block_tables, lens[k], w.scale, want_f64=True)
        assert_attention_close(outs[k], f64, what=f"pipelined host step {k}")
    torch.cuda.synchronize()
    assert torch.equal(a.k_cache.view(torch.int16), b.k_cache.view(torch.int16))
    assert pa.device_error() == 0
