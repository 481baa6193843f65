"""Randomised shapes through decode, the fused store + decode and prefill, against the oracle.

Every case draws its own group size, head dim, block size, context lengths (including 0 and 1), split size and
prefix; the seeds are fixed so any failure reproduces.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DeviceDecode, DevicePrefill, assert_attention_close

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("seed", range(12))
def test_decode_random_shapes(oracle, seed):
    rng = np.random.default_rng(5000 + seed)
    d = int(rng.choice([64, 128]))
    hkv = int(rng.integers(1, 5))
    g = int(rng.integers(1, 9))
    bs = int(rng.choice([16, 32, 64, 128, 256, 512, 1024]))
    B = int(rng.integers(1, 12))
    lens = rng.integers(0, 3000, B)
    lens[rng.random(B) < 0.15] = 1
    lens = lens.astype(np.int32)
    chunk = int(rng.choice([0, 64, 192, 1024]))
    w = W.decode_workload(lens, g * hkv, hkv, d, bs, rng=rng)
    a, b = DeviceDecode(w), DeviceDecode(w)
    L = int(max(1, lens.max()))
    out = pa.store_decode(a.q, a.new_k, a.new_v, a.slot_mapping, a.k_cache, a.v_cache, a.block_tables,
                          a.context_lens, L, w.scale, kv_chunk_size=chunk)
    pa.store_kvcache(b.new_k, b.new_v, b.k_cache, b.v_cache, b.slot_mapping)
    out2 = pa.decode(b.q, b.k_cache, b.v_cache, b.block_tables, b.context_lens, L, w.scale, kv_chunk_size=chunk)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), out2.view(torch.int16))
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what=f"decode seed {seed} (G={g} Hkv={hkv} D={d} bs={bs} chunk={chunk})")
    assert pa.device_error() == 0


@pytest.mark.parametrize("seed", range(10))
def test_prefill_random_shapes(oracle, seed):
    rng = np.random.default_rng(6000 + seed)
    d = int(rng.choice([64, 128]))
    hkv = int(rng.integers(1, 4))
    g = int(rng.choice([1, 2, 4, 8]))
    bs = int(rng.choice([16, 32, 64, 128, 256]))
    prefix = bs * int(rng.integers(0, 4))
    B = int(rng.integers(1, 6))
    sfx = [int(x) for x in rng.integers(0, 300, B)]
    sfx[0] = max(sfx[0], 1)
    causal = bool(rng.random() < 0.8)
    w = W.prefill_workload(prefix, sfx, g * hkv, hkv, d, bs, rng=rng, causal=causal)
    dw = DevicePrefill(w)
    pa.store_kvcache(dw.new_k, dw.new_v, dw.k_cache, dw.v_cache, dw.slot_mapping)
    out = pa.prefill_varlen(dw.q, dw.k_cache, dw.v_cache, dw.cu_seqlens_q, dw.cu_seqlens_k, w.max_seqlen_q,
                            w.max_seqlen_k, dw.block_tables, w.scale, causal)
    torch.cuda.synchronize()
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                   w.scale, causal, want_f64=True)
    assert_attention_close(out, ref, what=f"prefill seed {seed} (G={g} Hkv={hkv} D={d} bs={bs} prefix={prefix} "
                                          f"sfx={sfx} causal={causal})")
    assert pa.device_error() == 0
