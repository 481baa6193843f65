"""The split-KV chunk choice of pa_decode (host logic, CPU only), through
pa_decode_chunk_size_for: the choice pa_decode makes for a device with a given
number of SMs."""
import math

import numpy as np
import pytest

from paged_kv_cache_331_b200 import workloads as W

TILE, MIN_CHUNK, WAVES = 64, 512, 4


@pytest.fixture(scope="module")
def pa():
    from paged_kv_cache_331_b200 import build as B
    B.build()
    import paged_kv_cache_331_b200 as pa
    return pa


def test_invalid_arguments(pa):
    assert pa.decode_chunk_size_for(1, 1, 100, 0) == -1
    assert pa.decode_chunk_size_for(-1, 1, 100, 148) == -1
    assert pa.decode_chunk_size_for(1, 0, 100, 148) == -1
    assert pa.decode_chunk_size_for(1, 1, -5, 148) == -1


@pytest.mark.parametrize("sms", [1, 8, 132, 148])
def test_properties_over_a_grid(pa, sms):
    """Whole tiles; no split when short or already enough CTAs; otherwise at
    most ceil(L / 512) chunks and within one split of the wave target."""
    for units_seqs, hkv in ((1, 1), (1, 8), (3, 8), (9, 8), (64, 8), (256, 8), (2, 1), (500, 4)):
        units = units_seqs * hkv
        want = WAVES * 2 * sms
        for L in (0, 1, 63, 64, 100, 511, 512, 513, 1000, 1024, 2112, 4096, 5000, 32768, 131072):
            c = pa.decode_chunk_size_for(units_seqs, hkv, L, sms)
            assert c > 0 and c % TILE == 0, (units, L, sms, c)
            n = max(1, math.ceil(L / c))
            if L <= MIN_CHUNK or units >= want:
                assert n == 1 and c >= L, (units, L, sms, c)
                continue
            max_splits = math.ceil(L / MIN_CHUNK)
            target = min(max(math.ceil(want / units), 1), max_splits)
            assert n <= max_splits, (units, L, sms, c)
            # the chunk is the tile-rounded share of one of target - 1 .. target + 1 splits
            shares = {math.ceil(math.ceil(L / s) / TILE) * TILE for s in (target - 1, target, target + 1)
                      if 1 <= s <= max_splits}
            assert c in shares, (units, L, sms, c, shares)


def test_least_overhang_among_the_candidates(pa):
    """Of the candidate chunk sizes, the one chosen leaves the shortest idle
    tail behind the longest context; among equal tails, the fewest chunks."""
    sms = 148
    for units_seqs, hkv, L in ((9, 8, 32768), (4, 8, 10000), (2, 4, 7777), (16, 8, 3000), (1, 1, 100000)):
        units = units_seqs * hkv
        c = pa.decode_chunk_size_for(units_seqs, hkv, L, sms)
        overhang = math.ceil(L / c) * c - L
        max_splits = math.ceil(L / MIN_CHUNK)
        target = min(math.ceil(WAVES * 2 * sms / units), max_splits)
        for s in (target - 1, target, target + 1):
            if 1 <= s <= max_splits:
                alt = math.ceil(math.ceil(L / s) / TILE) * TILE
                alt_overhang = math.ceil(L / alt) * alt - L
                assert overhang <= alt_overhang, (units, L, c, alt)
                if overhang == alt_overhang:
                    assert c >= alt, (units, L, c, alt)


def test_bench_workloads_on_a_b200(pa):
    """The chunk sizes the B200 (148 SMs) gets for the measured workloads."""
    q = W.qwen3_decode()
    # 2 and 4 chunks overhang the longest context (4 068) equally; the tie goes to fewer CTAs
    assert pa.decode_chunk_size_for(q.num_seqs, q.num_kv_heads, q.max_context_len, 148) == 2048
    lc = W.long_context_decode()
    c = pa.decode_chunk_size_for(lc.num_seqs, lc.num_kv_heads, lc.max_context_len, 148)
    assert c == 2048 and lc.max_context_len // c == 16                 # 16-way split of 32k
    lb = W.large_batch_decode()
    assert pa.decode_chunk_size_for(lb.num_seqs, lb.num_kv_heads, lb.max_context_len, 148) >= lb.max_context_len


def test_workspace_follows_the_chunk(pa):
    """pa_decode_workspace_size with the chosen chunk is zero exactly when nothing is split."""
    for seqs, hkv, L in ((9, 8, 32768), (256, 8, 2048), (1, 8, 400), (4, 2, 9000)):
        c = pa.decode_chunk_size_for(seqs, hkv, L, 148)
        n = max(1, math.ceil(L / c))
        ws = pa.decode_workspace_size(seqs, hkv * 2, hkv, 128, L, 256, c)
        assert (ws == 0) == (n == 1)
        if n > 1:
            rows = seqs * hkv * 2 * n
            assert ws == (rows * 128 * 4 + 255) // 256 * 256 + rows * 2 * 4


def test_context_lengths_of_the_workloads_are_what_the_pins_assume():
    assert W.long_context_decode().max_context_len == 32768
    assert int(np.max(W.qwen3_decode().context_lens)) == W.qwen3_decode().max_context_len
