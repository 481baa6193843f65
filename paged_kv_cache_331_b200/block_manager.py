"""ctypes binding of the host-side block manager in libpagedattn.so
(``include/pa_block_manager.h``).

Argument marshalling only: every decision (prefix-cache lookups, reference
counts, block growth, slot arithmetic) is made by the C++ code.  Metadata comes
back as numpy int32 arrays in the layouts the attention entry points take.
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import _binding

_i32, _i64, _u64, _sz, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_uint64, ctypes.c_size_t, ctypes.c_void_p
_P32 = ctypes.POINTER(_i32)

_PROTOS = {
    "pa_xxh64": (_u64, [_vp, _sz, _u64]),
    "pa_bm_block_hash": (_u64, [_vp, _i32, _i32, _u64]),
    "pa_bm_create": (_vp, [_i32, _i32]),
    "pa_bm_destroy": (None, [_vp]),
    "pa_bm_num_free_blocks": (_i32, [_vp]),
    "pa_bm_add_sequence": (ctypes.c_int, [_vp, _i64, _vp, _i32]),
    "pa_bm_append_token": (ctypes.c_int, [_vp, _i64, _i32]),
    "pa_bm_remove_sequence": (ctypes.c_int, [_vp, _i64]),
    "pa_bm_can_allocate": (_i32, [_vp, _i64]),
    "pa_bm_allocate": (ctypes.c_int, [_vp, _i64]),
    "pa_bm_deallocate": (ctypes.c_int, [_vp, _i64]),
    "pa_bm_can_append": (_i32, [_vp, _i64]),
    "pa_bm_may_append": (ctypes.c_int, [_vp, _i64]),
    "pa_bm_sequence_info": (ctypes.c_int, [_vp, _i64, _P32, _P32, _P32]),
    "pa_bm_block_table": (ctypes.c_int, [_vp, _i64, _vp, _i32]),
    "pa_bm_block_info": (ctypes.c_int, [_vp, _i32, _P32, _P32, ctypes.POINTER(_u64)]),
    "pa_bm_prepare_prefill": (ctypes.c_int, [_vp, _vp, _i32, _i32, _i32, _vp, _vp, _vp, _vp, _vp, _P32]),
    "pa_bm_prepare_decode": (ctypes.c_int, [_vp, _vp, _i32, _i32, _vp, _vp, _vp, _vp]),
}
_ready = False


def _lib():
    global _ready
    L = _binding.lib()
    if not _ready:
        for name, (res, args) in _PROTOS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _ready = True
    return L


def _i32s(a) -> np.ndarray:
    return np.ascontiguousarray(a, dtype=np.int32)


def xxh64(data: bytes, seed: int = 0) -> int:
    return int(_lib().pa_xxh64(data, len(data), seed))


def block_hash(token_ids, prefix=None) -> int:
    t = _i32s(token_ids)
    return int(_lib().pa_bm_block_hash(t.ctypes.data, t.size, prefix is not None, 0 if prefix is None else prefix))


class BlockManager:
    """One manager of ``num_blocks`` cache blocks of ``block_size`` tokens."""

    def __init__(self, num_blocks: int, block_size: int):
        L = _lib()
        self._h = L.pa_bm_create(num_blocks, block_size)
        if not self._h:
            raise _binding.PagedAttentionError(f"pa_bm_create: {L.pa_last_error().decode()}")
        self.num_blocks, self.block_size = num_blocks, block_size

    def __del__(self):
        h = getattr(self, "_h", None)
        if h:
            self._h = None
            try:
                _lib().pa_bm_destroy(h)
            except Exception:     # interpreter shutdown: the library may already be gone
                pass

    def _ok(self, status, what):
        _binding._check(status, what)

    # sequences
    def add_sequence(self, seq_id: int, token_ids):
        t = _i32s(token_ids)
        self._ok(_lib().pa_bm_add_sequence(self._h, seq_id, t.ctypes.data, t.size), "pa_bm_add_sequence")

    def append_token(self, seq_id: int, token_id: int):
        self._ok(_lib().pa_bm_append_token(self._h, seq_id, int(token_id)), "pa_bm_append_token")

    def remove_sequence(self, seq_id: int):
        self._ok(_lib().pa_bm_remove_sequence(self._h, seq_id), "pa_bm_remove_sequence")

    # the block operations
    def can_allocate(self, seq_id: int) -> bool:
        r = _lib().pa_bm_can_allocate(self._h, seq_id)
        if r < 0:
            raise KeyError(seq_id)
        return bool(r)

    def allocate(self, seq_id: int):
        self._ok(_lib().pa_bm_allocate(self._h, seq_id), "pa_bm_allocate")

    def deallocate(self, seq_id: int):
        self._ok(_lib().pa_bm_deallocate(self._h, seq_id), "pa_bm_deallocate")

    def can_append(self, seq_id: int) -> bool:
        r = _lib().pa_bm_can_append(self._h, seq_id)
        if r < 0:
            raise KeyError(seq_id)
        return bool(r)

    def may_append(self, seq_id: int):
        self._ok(_lib().pa_bm_may_append(self._h, seq_id), "pa_bm_may_append")

    # introspection
    def num_free_blocks(self) -> int:
        return int(_lib().pa_bm_num_free_blocks(self._h))

    def sequence_info(self, seq_id: int):
        n, c, b = _i32(), _i32(), _i32()
        self._ok(_lib().pa_bm_sequence_info(self._h, seq_id, ctypes.byref(n), ctypes.byref(c), ctypes.byref(b)),
                 "pa_bm_sequence_info")
        return int(n.value), int(c.value), int(b.value)

    def block_table(self, seq_id: int) -> list:
        nb = self.sequence_info(seq_id)[2]
        out = np.zeros(max(nb, 1), np.int32)
        self._ok(_lib().pa_bm_block_table(self._h, seq_id, out.ctypes.data, out.size), "pa_bm_block_table")
        return out[:nb].tolist()

    def block_info(self, block_id: int):
        rc, hh, h = _i32(), _i32(), _u64()
        self._ok(_lib().pa_bm_block_info(self._h, block_id, ctypes.byref(rc), ctypes.byref(hh), ctypes.byref(h)),
                 "pa_bm_block_info")
        return int(rc.value), bool(hh.value), int(h.value)

    # batch metadata
    def prepare_prefill(self, seq_ids, max_blocks_per_seq: int, token_capacity: int | None = None) -> dict:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        B = ids.size
        if token_capacity is None:
            token_capacity = sum(self.sequence_info(int(s))[0] for s in ids)
        bt = np.empty((B, max_blocks_per_seq), np.int32)
        cq, ck = np.empty(B + 1, np.int32), np.empty(B + 1, np.int32)
        slots, pos = np.empty(max(token_capacity, 1), np.int32), np.empty(max(token_capacity, 1), np.int32)
        total = _i32()
        self._ok(_lib().pa_bm_prepare_prefill(self._h, ids.ctypes.data, B, max_blocks_per_seq, token_capacity,
                                              bt.ctypes.data, cq.ctypes.data, ck.ctypes.data, slots.ctypes.data,
                                              pos.ctypes.data, ctypes.byref(total)), "pa_bm_prepare_prefill")
        n = int(total.value)
        return dict(block_tables=bt, cu_seqlens_q=cq, cu_seqlens_k=ck, slot_mapping=slots[:n].copy(),
                    positions=pos[:n].copy())

    def prepare_decode(self, seq_ids, max_blocks_per_seq: int) -> dict:
        ids = np.ascontiguousarray(seq_ids, dtype=np.int64)
        B = ids.size
        bt = np.empty((B, max_blocks_per_seq), np.int32)
        ctx, slots, pos = (np.empty(B, np.int32) for _ in range(3))
        self._ok(_lib().pa_bm_prepare_decode(self._h, ids.ctypes.data, B, max_blocks_per_seq, bt.ctypes.data,
                                             ctx.ctypes.data, slots.ctypes.data, pos.ctypes.data),
                 "pa_bm_prepare_decode")
        return dict(block_tables=bt, context_lens=ctx, slot_mapping=slots, positions=pos)
