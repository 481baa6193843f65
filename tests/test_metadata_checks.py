"""Host checks of the device metadata the kernels take on trust (CPU only):
every workload passes, and each single violation is caught."""
import numpy as np
import pytest

from paged_kv_cache_331_b200 import workloads as W
from paged_kv_cache_331_b200.metadata import check_prefill_metadata, check_store_decode_metadata


def prefill_args(w):
    return dict(cu_seqlens_q=w.cu_seqlens_q.copy(), cu_seqlens_k=w.cu_seqlens_k.copy(),
                total_q=int(w.cu_seqlens_q[-1] - w.cu_seqlens_q[0]), max_seqlen_q=w.max_seqlen_q,
                max_seqlen_k=w.max_seqlen_k, block_tables=w.block_tables.copy(), block_size=w.block_size,
                num_blocks=w.k_cache.shape[0])


@pytest.fixture(scope="module")
def pw():
    return W.prefill_workload(32, np.array([9, 20, 0, 150], np.int32), 4, 2, 64, 16, rng=np.random.default_rng(3))


def test_prefill_workloads_pass(pw):
    check_prefill_metadata(**prefill_args(pw))
    check_prefill_metadata(**prefill_args(W.prefix_prefill()))


@pytest.mark.parametrize("mutate,match", [
    (lambda a: a.update(total_q=a["total_q"] + 1), "total_q"),
    (lambda a: a.update(max_seqlen_q=a["max_seqlen_q"] - 1), "max_seqlen_q"),
    (lambda a: a.update(max_seqlen_k=a["max_seqlen_k"] - 1), "max_seqlen_k"),
    (lambda a: a["cu_seqlens_k"].__setitem__(2, a["cu_seqlens_k"][1] - 1), "non-decreasing"),
    (lambda a: a["cu_seqlens_k"].__setitem__(slice(1, None), a["cu_seqlens_k"][1:] - 40), "fewer keys"),
    (lambda a: a["block_tables"].__setitem__((0, 1), -1), "not a block id"),
    (lambda a: a["block_tables"].__setitem__((3, 0), a["num_blocks"]), "not a block id"),
    (lambda a: a.update(block_tables=a["block_tables"][:, :3]), "table entries"),
    (lambda a: a.update(cu_seqlens_k=a["cu_seqlens_k"][:-1]), r"\[num_seqs \+ 1\]"),
])
def test_prefill_violations_are_caught(pw, mutate, match):
    a = prefill_args(pw)
    mutate(a)
    with pytest.raises(ValueError, match=match):
        check_prefill_metadata(**a)


def decode_args(w):
    return dict(slot_mapping=w.slot_mapping.copy(), block_tables=w.block_tables.copy(),
                context_lens=w.context_lens.copy(), max_context_len=w.max_context_len, block_size=w.block_size,
                num_blocks=w.k_cache.shape[0])


@pytest.fixture(scope="module")
def dw():
    return W.decode_workload(np.array([1, 17, 256, 300], np.int32), 4, 2, 64, 16, rng=np.random.default_rng(4))


def test_store_decode_workloads_pass(dw):
    check_store_decode_metadata(**decode_args(dw))
    check_store_decode_metadata(**decode_args(W.tiny_decode()))
    a = decode_args(dw)
    a["slot_mapping"][1] = -1                                     # nothing stored for that sequence
    check_store_decode_metadata(**a)


@pytest.mark.parametrize("mutate,match", [
    (lambda a: a["slot_mapping"].__setitem__(2, a["slot_mapping"][2] + 1), "slot_mapping\\[2\\]"),
    (lambda a: a["slot_mapping"].__setitem__(0, a["slot_mapping"][3]), "slot_mapping\\[0\\]"),
    (lambda a: a["block_tables"].__setitem__((3, 18), a["num_blocks"] + 5), "not a block id"),
    (lambda a: a["context_lens"].__setitem__(1, 0), "no position"),
    (lambda a: a.update(block_tables=a["block_tables"][:2]), "a row per sequence"),
])
def test_store_decode_violations_are_caught(dw, mutate, match):
    a = decode_args(dw)
    mutate(a)
    with pytest.raises(ValueError, match=match):
        check_store_decode_metadata(**a)
