"""Pins of the CPU oracle against things other than itself (no GPU).

Each pin is something the pages or mathematics fix independently of the
oracle's code: the page-table example printed in the lshu.cn essay (§3.2),
torch's own scaled_dot_product_attention / causal_lower_right in float64,
closed forms (one key, equal keys, one dominant key), invariances (physical
block permutation, shared vs duplicated prefix blocks), and torch's float ->
bf16 rounding.
"""
import math

import numpy as np
import pytest
import torch

from conftest import read_golden
from attn_ref import decode_reference, prefill_reference, gather_contiguous
from paged_kv_cache_331_b200 import workloads as W

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


def store_new_rows(oracle, w):
    oracle.store_kvcache(w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)


def small_decode(seed, lens, hq=4, hkv=2, d=64, bs=16, **kw):
    rng = np.random.default_rng(seed)
    return W.decode_workload(np.asarray(lens, np.int32), hq, hkv, d, bs, rng=rng, **kw)


def permute_pool(w, seed):
    """Same logical contents under a different physical block assignment."""
    rng = np.random.default_rng(seed)
    pi = rng.permutation(w.num_blocks).astype(np.int32)
    kc = np.empty_like(w.k_cache); vc = np.empty_like(w.v_cache)
    kc[pi] = w.k_cache; vc[pi] = w.v_cache
    bt = np.where(w.block_tables >= 0, pi[np.maximum(w.block_tables, 0)], -1).astype(np.int32)
    return kc, vc, bt


# ---------------------------------------------------------------------------- address math ---

def test_page_table_worked_example(oracle):
    (g,) = read_golden("page_table_example.txt")
    table = np.array([[11, 5, 7], [2, 3, 4]], dtype=np.int32)   # arbitrary physical pages of two requests
    blk, off = oracle.kv_location(table, 0, g["position"], g["page_size"], 16)
    assert blk == table[0, g["page_index"]]
    assert off == g["offset"]


def test_store_then_gather_round_trip(oracle):
    """Rows scattered through slot_mapping come back bit-exactly through the page-table walk."""
    rng = np.random.default_rng(7)
    for bs in (16, 256):
        nb, hkv, d = 12, 2, 64
        kc = np.full((nb, bs, hkv, d), 0x3F80, np.uint16)
        vc = np.full((nb, bs, hkv, d), 0x3F80, np.uint16)
        table = rng.permutation(nb)[None, :5].astype(np.int32)
        n = 3 * bs + 5
        pos = np.arange(n)
        slots = W.slots_for_positions(table[0], pos, bs)
        key = W.randn_bf16(rng, (n, hkv, d)); val = W.randn_bf16(rng, (n, hkv, d))
        oracle.store_kvcache(key, val, kc, vc, slots)
        for p in (0, 1, bs - 1, bs, 2 * bs + 3, n - 1):
            blk, off = oracle.kv_location(table, 0, p, bs, nb)
            assert np.array_equal(kc[blk, off], key[p]) and np.array_equal(vc[blk, off], val[p])
        # every other row still holds the sentinel
        assert int((kc != 0x3F80).any(axis=(2, 3)).sum()) == n


def test_store_skips_minus_one_and_touches_nothing_else(oracle):
    rng = np.random.default_rng(8)
    nb, bs, hkv, d = 4, 16, 2, 64
    kc = W.randn_bf16(rng, (nb, bs, hkv, d)); vc = W.randn_bf16(rng, (nb, bs, hkv, d))
    k0, v0 = kc.copy(), vc.copy()
    key = W.randn_bf16(rng, (5, hkv, d)); val = W.randn_bf16(rng, (5, hkv, d))
    slots = np.array([-1, 17, -1, 0, 63], np.int32)
    oracle.store_kvcache(key, val, kc, vc, slots)
    kf, vf = kc.reshape(nb * bs, hkv, d), vc.reshape(nb * bs, hkv, d)
    for t, s in enumerate(slots):
        if s >= 0:
            assert np.array_equal(kf[s], key[t]) and np.array_equal(vf[s], val[t])
    untouched = np.setdiff1d(np.arange(nb * bs), slots[slots >= 0])
    assert np.array_equal(kf[untouched], k0.reshape(nb * bs, hkv, d)[untouched])
    assert np.array_equal(vf[untouched], v0.reshape(nb * bs, hkv, d)[untouched])
    # all slots -1: the cache is byte-identical
    kc2, vc2 = k0.copy(), v0.copy()
    oracle.store_kvcache(key, val, kc2, vc2, np.full(5, -1, np.int32))
    assert kc2.tobytes() == k0.tobytes() and vc2.tobytes() == v0.tobytes()


def test_store_strided_rows(oracle):
    """key/value may be views into a fused qkv buffer (row stride > Hkv*D)."""
    rng = np.random.default_rng(9)
    hq, hkv, d, n = 4, 2, 64, 6
    qkv = W.randn_bf16(rng, (n, (hq + 2 * hkv) * d))
    key = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d)
    val = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d)
    kc = np.zeros((2, 16, hkv, d), np.uint16); vc = np.zeros_like(kc)
    slots = np.array([3, 4, 5, 16, 17, 31], np.int32)
    oracle.store_kvcache(key, val, kc, vc, slots)
    assert np.array_equal(kc.reshape(32, hkv, d)[slots], key)
    assert np.array_equal(vc.reshape(32, hkv, d)[slots], val)


# ------------------------------------------------------------------------------- bf16 rounding ---

def test_bf16_rounding_matches_torch(oracle):
    """double -> bf16 of float32-representable values equals torch's float32 -> bf16 (RNE)."""
    rng = np.random.default_rng(10)
    x = rng.standard_normal(20000).astype(np.float32) * np.float32(3.0)
    # exact ties between two bf16 neighbours, both parities, and tiny / huge magnitudes
    base = W.bf16_bits_to_f32(rng.integers(0x3000, 0x5000, 2000).astype(np.uint16))
    ulp = np.ldexp(np.float32(1), np.frexp(base)[1] - 8).astype(np.float32)
    ties = (base + ulp / 2).astype(np.float32)
    extra = np.array([1e-38, -1e-39, 3.3e38, -3.39e38, 0.0, -0.0, 1.0], np.float32)
    x = np.concatenate([x, ties, -ties, extra])
    got = oracle.bf16_round(x.astype(np.float64))
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, want)


# --------------------------------------------------------------------------------------- decode ---

@pytest.mark.parametrize("lens,hq,hkv,d,bs", [
    ([1, 17, 256, 300], 4, 2, 64, 256),
    ([5, 33, 64, 1, 100], 8, 2, 128, 16),
    ([40, 41], 4, 4, 64, 32),
    ([129, 7], 8, 1, 64, 64),
])
def test_decode_matches_torch_sdpa(oracle, lens, hq, hkv, d, bs):
    w = small_decode(11, lens, hq, hkv, d, bs)
    store_new_rows(oracle, w)
    out, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    ref = decode_reference(w)
    np.testing.assert_allclose(of, ref, rtol=0, atol=1e-12)
    assert np.array_equal(out, oracle.bf16_round(of))


def test_tiny_decode_workload_matches_sdpa(oracle):
    w = W.tiny_decode()
    store_new_rows(oracle, w)
    _, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    np.testing.assert_allclose(of, decode_reference(w), rtol=0, atol=1e-12)


def test_decode_block_permutation_invariance(oracle):
    w = small_decode(12, [70, 3, 48, 16], bs=16)
    store_new_rows(oracle, w)
    a = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    kc, vc, bt = permute_pool(w, 99)
    b = oracle.decode(w.q, kc, vc, bt, w.context_lens, w.scale)
    assert np.array_equal(a, b)


def test_decode_single_key_returns_value_row(oracle):
    """L = 1: softmax over one key is 1, so o is that V row exactly."""
    w = small_decode(13, [1, 1, 1], hq=4, hkv=2, bs=16)
    store_new_rows(oracle, w)
    out = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    for b in range(3):
        for h in range(4):
            assert np.array_equal(out[b, h], w.new_v[b, h // 2])


def test_decode_equal_keys_give_mean_value(oracle):
    """All keys equal => uniform weights => o is the mean of the V rows (closed form)."""
    w = small_decode(14, [37, 16], hq=4, hkv=2, bs=16)
    w.k_cache[:] = w.k_cache[0, 0]
    out, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    for b, L in enumerate(w.context_lens):
        v = gather_contiguous(w.v_cache, w.block_tables[b], int(L), w.block_size).numpy()
        for h in range(4):
            np.testing.assert_allclose(of[b, h], v[:, h // 2].mean(axis=0), rtol=0, atol=1e-13)


def test_decode_dominant_key_selects_its_value(oracle):
    """One key aligned with q and 60x larger than the rest: its weight is 1 to within 1e-12."""
    w = small_decode(15, [50], hq=2, hkv=1, d=64, bs=16)
    q = W.bf16_bits_to_f32(w.q[0, 0])
    w.q[0, 1] = w.q[0, 0]
    w.k_cache[:] = 0
    j = 23
    blk, off = w.block_tables[0, j // 16], j % 16
    w.k_cache[blk, off, 0] = W.f32_to_bf16_bits(np.sign(q) * 2.0)
    w.scale = 1.0
    _, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, 1.0, want_f64=True)
    vj = W.bf16_bits_to_f32(w.v_cache[blk, off, 0]).astype(np.float64)
    np.testing.assert_allclose(of[0, 0], vj, atol=1e-12 * 50 * 10)


def test_decode_zero_context_gives_zero(oracle):
    w = small_decode(16, [0, 5], bs=16)
    out = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    assert not out[0].any()


def test_decode_ignores_poisoned_rows(oracle):
    """NaN in every cache row outside the contexts changes nothing."""
    w = small_decode(17, [70, 3, 48, 16], bs=16)
    store_new_rows(oracle, w)
    clean = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    W._poison_outside_context(w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.block_size)
    dirty = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale)
    assert np.array_equal(clean, dirty)


def test_decode_brute_force_tiny(oracle):
    """Pure-Python exhaustive evaluation with math.fsum on a 2-sequence, block-size-4 case."""
    w = small_decode(18, [3, 6], hq=2, hkv=1, d=8, bs=4, pool_blocks=5)
    store_new_rows(oracle, w)
    _, of = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    f = lambda a: [float(x) for x in W.bf16_bits_to_f32(a)]
    for b in range(2):
        L = int(w.context_lens[b])
        keys = [f(w.k_cache[w.block_tables[b, j // 4], j % 4, 0]) for j in range(L)]
        vals = [f(w.v_cache[w.block_tables[b, j // 4], j % 4, 0]) for j in range(L)]
        for h in range(2):
            q = f(w.q[b, h])
            logits = [w.scale * math.fsum(qq * kk for qq, kk in zip(q, k)) for k in keys]
            mx = max(logits)
            e = [math.exp(s - mx) for s in logits]
            z = math.fsum(e)
            want = [math.fsum(e[j] * vals[j][d] for j in range(L)) / z for d in range(8)]
            np.testing.assert_allclose(of[b, h], want, rtol=0, atol=1e-13)


@pytest.mark.parametrize("chunk", [1, 16, 48, 64, 1000])
def test_split_merge_identity(oracle, chunk):
    """Log-sum-exp merge of per-chunk partials equals the unsplit result for any chunking."""
    w = small_decode(19, [70, 3, 48, 16, 0], bs=16)
    store_new_rows(oracle, w)
    _, whole = oracle.decode(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    nch = max(1, math.ceil(int(w.context_lens.max()) / chunk))
    m, l, acc = oracle.decode_partials(w.q, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, chunk, nch)
    _, merged = oracle.merge_partials(m, l, acc)
    np.testing.assert_allclose(merged, whole, rtol=0, atol=1e-12)


# -------------------------------------------------------------------------------------- prefill ---

def small_prefill(seed, prefix, sfx, hq=4, hkv=2, d=64, bs=16, **kw):
    rng = np.random.default_rng(seed)
    return W.prefill_workload(prefix, np.asarray(sfx, np.int32), hq, hkv, d, bs, rng=rng, **kw)


@pytest.mark.parametrize("prefix,sfx,causal,hq,hkv,d,bs", [
    (0, [5, 17, 1], True, 4, 2, 64, 16),        # no prefix: plain causal
    (32, [5, 17, 1], True, 4, 2, 64, 16),       # shared prefix, bottom-right causal
    (32, [9, 20], False, 4, 1, 128, 16),        # non-causal
    (64, [40, 3], True, 8, 2, 128, 32),
])
def test_prefill_matches_torch_sdpa(oracle, prefix, sfx, causal, hq, hkv, d, bs):
    w = small_prefill(21, prefix, sfx, hq, hkv, d, bs, causal=causal)
    store_new_rows(oracle, w)
    out, of = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                    w.scale, w.causal, want_f64=True)
    np.testing.assert_allclose(of, prefill_reference(w), rtol=0, atol=1e-12)


def test_prefill_rows_equal_decode(oracle):
    """Prefill row i of a sequence equals a decode step with context Lk - Lq + i + 1 on the same table."""
    w = small_prefill(22, 32, [7, 12], bs=16)
    store_new_rows(oracle, w)
    out = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables,
                                w.scale, True)
    for b in range(2):
        q0, q1 = w.cu_seqlens_q[b], w.cu_seqlens_q[b + 1]
        Lq, Lk = q1 - q0, w.cu_seqlens_k[b + 1] - w.cu_seqlens_k[b]
        for i in range(Lq):
            d = oracle.decode(w.q[q0 + i:q0 + i + 1], w.k_cache, w.v_cache, w.block_tables[b:b + 1],
                              np.array([Lk - Lq + i + 1], np.int32), w.scale)
            assert np.array_equal(d[0], out[q0 + i])


def test_prefill_shared_vs_duplicated_prefix(oracle):
    """Prefix blocks shared by reference give the same output as private copies of them."""
    a = small_prefill(23, 48, [9, 20, 4], bs=16, shared_prefix=True)
    b = small_prefill(23, 48, [9, 20, 4], bs=16, shared_prefix=False)
    # same logical contents: copy a's per-position rows into b's layout
    for s in range(a.num_seqs):
        Lk = int(a.cu_seqlens_k[s + 1] - a.cu_seqlens_k[s])
        for p in range(Lk):
            b.k_cache[b.block_tables[s, p // 16], p % 16] = a.k_cache[a.block_tables[s, p // 16], p % 16]
            b.v_cache[b.block_tables[s, p // 16], p % 16] = a.v_cache[a.block_tables[s, p // 16], p % 16]
    b.q[:] = a.q; b.new_k[:] = a.new_k; b.new_v[:] = a.new_v
    assert len(np.unique(a.block_tables[:, :3])) == 3 and len(np.unique(b.block_tables[:, :3])) == 9
    for w in (a, b):
        store_new_rows(oracle, w)
    oa = oracle.prefill_varlen(a.q, a.k_cache, a.v_cache, a.cu_seqlens_q, a.cu_seqlens_k, a.block_tables, a.scale)
    ob = oracle.prefill_varlen(b.q, b.k_cache, b.v_cache, b.cu_seqlens_q, b.cu_seqlens_k, b.block_tables, b.scale)
    assert np.array_equal(oa, ob)


def test_prefill_permutation_and_poison_invariance(oracle):
    w = small_prefill(24, 32, [9, 20], bs=16)
    store_new_rows(oracle, w)
    base = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables, w.scale)
    kc, vc, bt = permute_pool(w, 5)
    perm = oracle.prefill_varlen(w.q, kc, vc, w.cu_seqlens_q, w.cu_seqlens_k, bt, w.scale)
    assert np.array_equal(base, perm)
    W._poison_outside_context(kc, vc, bt, np.diff(w.cu_seqlens_k), 16)
    pois = oracle.prefill_varlen(w.q, kc, vc, w.cu_seqlens_q, w.cu_seqlens_k, bt, w.scale)
    assert np.array_equal(base, pois)


def test_prefill_row_select_computes_only_selected(oracle):
    w = small_prefill(25, 16, [6, 5], bs=16)
    store_new_rows(oracle, w)
    full = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables, w.scale)
    sel = np.zeros(11, np.uint8); sel[[0, 4, 6, 10]] = 1
    part = oracle.prefill_varlen(w.q, w.k_cache, w.v_cache, w.cu_seqlens_q, w.cu_seqlens_k, w.block_tables, w.scale,
                                 row_select=sel)
    assert np.array_equal(part[sel == 1], full[sel == 1])
    assert not part[sel == 0].any()
