"""Host checks of the device metadata the kernels are given (``include/pa.h``).

The C ABI cannot read device arrays without synchronising, so the kernels
check this metadata themselves: a violation is skipped or clamped on the
device and reported through the device error word, after the launch:

- ``pa_prefill_varlen`` needs ``cu_seqlens_q/k`` to agree with ``total_q``,
  ``max_seqlen_q/k`` and the width of the block tables (a sequence that does
  not is skipped, code 8);
- ``pa_store_decode`` writes the new row at the slot the block table names for
  position ``L - 1`` (another slot is not written, code 5; a block id outside
  the cache neither, code 6).

These functions check the same rules on host copies of the arrays before
anything is launched and raise ``ValueError`` naming the first violation.  The
Python binding runs them when a call passes ``validate=True`` (which
synchronises); a caller that builds its metadata on the host can run them
before uploading.
"""
from __future__ import annotations

import numpy as np


def _host(a) -> np.ndarray:
    if hasattr(a, "detach"):
        a = a.detach().cpu().numpy()
    return np.asarray(a)


def _check_table_entries(tables: np.ndarray, lengths: np.ndarray, block_size: int, num_blocks: int, what: str):
    for b, n in enumerate(lengths):
        nblk = -(-int(n) // block_size)
        if nblk > tables.shape[1]:
            raise ValueError(f"{what}: sequence {b} needs {nblk} table entries, the tables have {tables.shape[1]}")
        ids = tables[b, :nblk]
        bad = np.nonzero((ids < 0) | (ids >= num_blocks))[0]
        if bad.size:
            raise ValueError(f"{what}: block_tables[{b}][{int(bad[0])}] = {int(ids[bad[0]])} is not a block id "
                             f"in [0, {num_blocks})")


def check_prefill_metadata(cu_seqlens_q, cu_seqlens_k, total_q: int, max_seqlen_q: int, max_seqlen_k: int,
                           block_tables, block_size: int, num_blocks: int) -> None:
    """The preconditions of pa_prefill_varlen on its device metadata."""
    cq, ck = _host(cu_seqlens_q).astype(np.int64), _host(cu_seqlens_k).astype(np.int64)
    bt = _host(block_tables)
    if cq.ndim != 1 or cq.size < 1 or ck.shape != cq.shape:
        raise ValueError("prefill: cu_seqlens_q and cu_seqlens_k must both be [num_seqs + 1]")
    lq, lk = np.diff(cq), np.diff(ck)
    if (lq < 0).any() or (lk < 0).any():
        raise ValueError("prefill: cu_seqlens_q and cu_seqlens_k must be non-decreasing")
    if int(cq[-1] - cq[0]) != int(total_q):
        raise ValueError(f"prefill: cu_seqlens_q spans {int(cq[-1] - cq[0])} rows, total_q is {total_q}")
    if lq.size and int(lq.max()) > max_seqlen_q:
        raise ValueError(f"prefill: a sequence has {int(lq.max())} query tokens, max_seqlen_q is {max_seqlen_q}")
    if lk.size and int(lk.max()) > max_seqlen_k:
        raise ValueError(f"prefill: a sequence has {int(lk.max())} keys, max_seqlen_k is {max_seqlen_k}")
    short = np.nonzero(lk < lq)[0]
    if short.size:
        raise ValueError(f"prefill: sequence {int(short[0])} has fewer keys than query tokens")
    if bt.ndim != 2 or bt.shape[0] < lq.size:
        raise ValueError("prefill: block_tables must be [num_seqs, max_blocks_per_seq]")
    _check_table_entries(bt, lk, block_size, num_blocks, "prefill")


def check_store_decode_metadata(slot_mapping, block_tables, context_lens, max_context_len: int, block_size: int,
                                num_blocks: int) -> None:
    """The preconditions of pa_store_decode: every slot is -1 or the slot that sequence b's table names for its
    newest position context_lens[b] - 1, through a valid block id."""
    slots, bt, lens = _host(slot_mapping).astype(np.int64), _host(block_tables), _host(context_lens).astype(np.int64)
    B = slots.size
    if lens.size < B or bt.ndim != 2 or bt.shape[0] < B:
        raise ValueError("store_decode: block_tables and context_lens need a row per sequence")
    lens = np.minimum(lens[:B], max_context_len)
    _check_table_entries(bt[:B], lens, block_size, num_blocks, "store_decode")
    for b in range(B):
        if slots[b] == -1:
            continue
        L = int(lens[b])
        if L <= 0:
            raise ValueError(f"store_decode: sequence {b} has no position to store (context length {L})")
        pos = L - 1
        expect = int(bt[b, pos // block_size]) * block_size + pos % block_size
        if slots[b] != expect:
            raise ValueError(f"store_decode: slot_mapping[{b}] = {int(slots[b])}, position {pos} of its table is "
                             f"slot {expect}")
