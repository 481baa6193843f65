"""Paged GQA decode (and its split-KV merge) on the GPU against the oracle."""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DeviceDecode, assert_attention_close, dev_bf16, dev_i32, host_bits

pytestmark = pytest.mark.gpu


def store_and_decode(dw, kv_chunk_size=0):
    w = dw.w
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    out = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, w.max_context_len, w.scale,
                    kv_chunk_size=kv_chunk_size)
    torch.cuda.synchronize()
    return out


def oracle_decode(oracle, w):
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    return of


CASES = [
    # lens, hq, hkv, d, bs
    ([1, 17, 256, 300], 4, 2, 64, 256),
    ([5, 33, 64, 1, 100, 0, 129], 8, 2, 128, 16),
    ([200, 64, 65, 63], 3, 1, 128, 32),
    ([700, 1], 5, 1, 64, 64),
    ([333, 1000, 2], 8, 1, 128, 128),
    ([1500, 257], 16, 2, 128, 1024),
    ([90, 91, 92], 6, 1, 64, 16),
    ([130, 7], 7, 1, 128, 256),
    ([640, 100], 2, 2, 64, 512),
]


@pytest.mark.parametrize("lens,hq,hkv,d,bs", CASES)
@pytest.mark.parametrize("chunk", [0, 64, 192, 512])
def test_decode_small_shapes(oracle, lens, hq, hkv, d, bs, chunk):
    rng = np.random.default_rng(sum(lens) + hq * 7 + d + bs)
    w = W.decode_workload(np.array(lens, np.int32), hq, hkv, d, bs, rng=rng)
    out = store_and_decode(DeviceDecode(w), kv_chunk_size=chunk)
    ref = oracle_decode(oracle, w)
    assert_attention_close(out, ref, what=f"decode {lens} G={hq // hkv} D={d} bs={bs} chunk={chunk}")
    zero_rows = np.asarray(lens) == 0
    if zero_rows.any():
        assert not host_bits(out)[zero_rows].any()


@pytest.mark.parametrize("make", [W.tiny_decode, W.qwen3_decode, W.large_batch_decode, W.long_context_decode])
def test_decode_named_workloads_full_size(oracle, make):
    """Every output element of the full-size workloads, automatic split-KV."""
    w = make()
    dw = DeviceDecode(w)
    out = store_and_decode(dw)
    ref = oracle_decode(oracle, w)
    mx, mean = assert_attention_close(out, ref, what=w.name)
    print(f"{w.name}: chunk={pa.decode_chunk_size(w.num_seqs, w.num_kv_heads, w.max_context_len, w.block_size)} "
          f"max_abs={mx:.2e} mean_abs={mean:.2e}")


def test_decode_poisoned_cache_and_determinism(oracle):
    """NaN in every cache row outside the contexts (and in unused blocks) changes nothing; repeat runs are
    bitwise identical."""
    rng = np.random.default_rng(31)
    lens = np.array([700, 3, 129, 64, 1, 250], np.int32)
    w = W.decode_workload(lens, 8, 2, 128, 64, rng=rng, poison_unused=True)
    # the new rows are stored into poisoned slots first
    dw = DeviceDecode(w)
    out1 = store_and_decode(dw, kv_chunk_size=128)
    out2 = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, w.max_context_len, w.scale,
                     kv_chunk_size=128)
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    ref = oracle_decode(oracle, w)
    assert_attention_close(out1, ref, what="poisoned")


def test_decode_block_table_padding_never_read(oracle):
    """Entries past ceil(L / block_size) hold -1 (and the table is wider than needed)."""
    rng = np.random.default_rng(32)
    w = W.decode_workload(np.array([40, 17], np.int32), 4, 2, 64, 16, rng=rng)
    wide = np.full((2, 64), -1, np.int32)
    wide[:, :w.block_tables.shape[1]] = w.block_tables
    w.block_tables = wide
    out = store_and_decode(DeviceDecode(w))
    assert_attention_close(out, oracle_decode(oracle, w), what="padded table")


def test_decode_workspace_too_small_is_rejected():
    rng = np.random.default_rng(33)
    w = W.decode_workload(np.array([1000], np.int32), 4, 2, 64, 16, rng=rng)
    dw = DeviceDecode(w)
    need = pa.decode_workspace_size(1, 4, 2, 64, 1000, 16, 64)
    assert need > 0
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(pa.PagedAttentionError, match="WORKSPACE"):
        pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 1000, w.scale,
                  kv_chunk_size=64, workspace=small)


def test_decode_no_device_error():
    assert pa.device_error() == 0


def test_decode_empty_batch():
    q = torch.empty(0, 4, 64, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(2, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    bt = torch.empty(0, 1, dtype=torch.int32, device="cuda")
    cl = torch.empty(0, dtype=torch.int32, device="cuda")
    out = pa.decode(q, kc, kc, bt, cl, 0, 0.125)
    o, lse = pa.decode_partial(q, kc, kc, bt, cl, 0, 0.125)
    torch.cuda.synchronize()
    assert out.shape == (0, 4, 64) and o.shape == (0, 4, 64) and lse.shape == (0, 4)
    assert pa.device_error() == 0


@pytest.mark.parametrize("chunk", [0, 128])
@pytest.mark.parametrize("n", [512, 600])
def test_decode_many_sequences_in_and_past_the_longest_first_range(oracle, n, chunk):
    """Up to 512 sequences per launch the CTAs take the longest sequences first (the first CTA ranks the context
    lengths and tells every other CTA its sequence); above that they follow the sequence index.  Both sides of
    the limit, with ties in length and empty sequences, unsplit and split into 128-token chunks, against the
    oracle (the fused store included)."""
    rng = np.random.default_rng(800 + n)
    lens = rng.integers(0, 300, n).astype(np.int32)
    lens[::7] = 128                                      # ties
    lens[::11] = 0                                       # empty sequences
    w = W.decode_workload(lens, 4, 2, 64, 64, rng=rng)
    dw = DeviceDecode(w)
    out = pa.store_decode(dw.q, dw.new_k, dw.new_v, dw.slot_mapping, dw.k_cache, dw.v_cache, dw.block_tables,
                          dw.context_lens, int(lens.max()), w.scale, kv_chunk_size=chunk)
    torch.cuda.synchronize()
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what=f"decode of {n} sequences, chunk {chunk}")
    assert pa.device_error() == 0


def test_decode_at_the_sequence_limit(oracle):
    """65 535 sequences in one launch (the most the grid's z dimension holds): index-order dispatch, contexts of
    1..200 tokens over 64-token blocks, split into 64-token chunks so that the separate merge kernel runs (more
    than 16 384 sequence x kv-head pairs), and unsplit, against the oracle."""
    n = 65535
    rng = np.random.default_rng(65535)
    lens = rng.integers(1, 201, n).astype(np.int32)
    w = W.decode_workload(lens, 2, 1, 64, 64, rng=rng)
    dw = DeviceDecode(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    out = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 200, w.scale, kv_chunk_size=64)
    whole = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 200, w.scale)
    torch.cuda.synchronize()
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what="decode of 65 535 sequences")
    assert_attention_close(whole, ref, what="decode of 65 535 sequences, automatic chunk")
    assert pa.device_error() == 0


def test_decode_one_very_long_context(oracle):
    """One sequence of 524 288 tokens (2 048 blocks of 256): the automatic split cuts it into 1 024 chunks whose
    partials the last chunk's CTA merges, against the oracle; plus a second, short sequence."""
    rng = np.random.default_rng(524288)
    lens = np.array([524288, 5], np.int32)
    w = W.decode_workload(lens, 8, 1, 128, 256, rng=rng)
    dw = DeviceDecode(w)
    chunk = pa.decode_chunk_size(2, 1, int(lens.max()), 256)
    assert -(-int(lens.max()) // chunk) >= 512
    out = pa.store_decode(dw.q, dw.new_k, dw.new_v, dw.slot_mapping, dw.k_cache, dw.v_cache, dw.block_tables,
                          dw.context_lens, int(lens.max()), w.scale)
    torch.cuda.synchronize()
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what="decode of a 524 288-token context")
    assert pa.device_error() == 0


@pytest.mark.parametrize("seed", range(12))
def test_dispatch_order_fuzz(oracle, seed):
    """Random shapes across the dispatch paths (unsplit or split, first waves of many or of one sequence
    position, empty sequences, the longest sequence anywhere): three launches in a row, each with the fused
    store of a fresh row, against the oracle's store + decode chain."""
    rng = np.random.default_rng(9000 + seed)
    hkv = int(rng.choice([1, 2, 4, 8]))
    g = int(rng.choice([1, 2, 4]))
    d = int(rng.choice([64, 128]))
    bs = int(rng.choice([16, 64, 256]))
    n = int(rng.integers(2, 48))
    lens = rng.integers(0, int(rng.choice([300, 2000, 6000])), n).astype(np.int32)
    lens[rng.integers(0, n)] = lens.max() + int(rng.integers(1, 200))      # a longest sequence, anywhere
    chunk = int(rng.choice([0, 64, 128, 512]))
    w = W.decode_workload(lens + 3, hkv * g, hkv, d, bs, rng=rng)              # room for three new tokens
    dw = DeviceDecode(w)
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    cur = lens.copy()
    for step in range(3):
        cur = cur + 1
        slots = np.array([W.slots_for_positions(w.block_tables[b], [int(cur[b]) - 1], bs)[0] for b in range(n)],
                         np.int32)
        new_k = W.randn_bf16(rng, (n, hkv, d))
        new_v = W.randn_bf16(rng, (n, hkv, d))
        cl = torch.from_numpy(cur).to(dw.q.device)
        out = pa.store_decode(dw.q, dev_bf16(new_k), dev_bf16(new_v), dev_i32(slots), dw.k_cache, dw.v_cache,
                              dw.block_tables, cl, int(cur.max()), w.scale, kv_chunk_size=chunk)
        torch.cuda.synchronize()
        oracle.store_kvcache(new_k, new_v, kc, vc, slots)
        _, ref = oracle.decode(w.q, kc, vc, w.block_tables, cur, w.scale, want_f64=True)
        assert_attention_close(out, ref, what=f"seed {seed} step {step} (hkv {hkv}, g {g}, d {d}, bs {bs}, "
                                              f"n {n}, chunk {chunk})")
    assert pa.device_error() == 0


def test_longest_first_when_one_position_fills_a_wave(oracle):
    """A split launch whose kv heads x chunks at one sequence position are more CTAs than one wave holds (64
    chunks x 8 kv heads): the first CTA, which sorts the other sequences, keeps sequence 0 at position 0, and
    the longest sequence (the second) is placed after it.  Twenty launches in a row, each against the oracle,
    so that merge counters left behind by one launch would show in the next."""
    rng = np.random.default_rng(4096)
    lens = np.array([100, 4096, 3000], np.int32)
    w = W.decode_workload(lens, 16, 8, 128, 256, rng=rng)
    dw = DeviceDecode(w)
    chunk = 64
    assert -(-int(lens.max()) // chunk) * 8 > 2 * 148
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    for i in range(20):
        out = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, int(lens.max()), w.scale,
                        kv_chunk_size=chunk)
        torch.cuda.synchronize()
        assert_attention_close(out, ref, what=f"launch {i}")
    assert pa.device_error() == 0


@pytest.mark.parametrize("chunk", [1024, 256])
def test_longest_first_order_is_repeatable_and_graph_safe(oracle, chunk):
    """The dispatch order lives in per-slot device entries that every launch leaves clean: many launches in a
    row (more than the 16 slots), and replays of one captured graph with changing context lengths, all give
    bitwise the same output as a fresh eager call on the same inputs; unsplit (1024-token chunks) and split
    into up to four chunks merged in the kernel (256)."""
    rng = np.random.default_rng(1717)
    w = W.decode_workload(np.full(96, 900, np.int32), 16, 8, 128, 256, rng=rng)   # tables cover 900 tokens
    lens = rng.integers(1, 900, 96).astype(np.int32)
    dw = DeviceDecode(w)
    dw.context_lens.copy_(torch.from_numpy(lens))
    first = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 900, w.scale,
                      kv_chunk_size=chunk)
    for _ in range(40):
        again = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, 900, w.scale,
                          kv_chunk_size=chunk)
    torch.cuda.synchronize()
    assert torch.equal(first.view(torch.int16), again.view(torch.int16))
    out = torch.empty_like(dw.q)
    cl = dw.context_lens.clone()
    assert (pa.decode_workspace_size(96, 16, 8, 128, 900, 256, chunk) == 0) == (chunk >= 900)
    ws = torch.empty(max(16, pa.decode_workspace_size(96, 16, 8, 128, 900, 256, chunk)), dtype=torch.uint8,
                     device=dw.q.device)
    pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, cl, 900, w.scale, out=out, workspace=ws,
              kv_chunk_size=chunk)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, cl, 900, w.scale, out=out, workspace=ws,
                  kv_chunk_size=chunk)
    for trial in range(3):
        new_lens = rng.integers(1, 900, 96).astype(np.int32)
        cl.copy_(torch.from_numpy(new_lens))
        g.replay()
        eager = pa.decode(dw.q, dw.k_cache, dw.v_cache, dw.block_tables, cl, 900, w.scale, kv_chunk_size=chunk)
        torch.cuda.synchronize()
        assert torch.equal(out.view(torch.int16), eager.view(torch.int16)), trial
        _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, new_lens, w.scale, want_f64=True)
        assert_attention_close(out, ref, what=f"graph replay {trial} with new context lengths")
    assert pa.device_error() == 0
