"""numpy-facing wrapper of the C oracle -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It compiles ``oracle.c`` with gcc into
``liboracle.so`` beside it (or a planted-mistake variant, for the tests that
show each pin catches a plausible error) and marshals numpy arrays into it.
bf16 tensors are ``uint16`` bit patterns.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from pathlib import Path

import numpy as np

HERE = Path(__file__).resolve().parent
SRC = HERE / "oracle.c"

_c_i32p = ctypes.POINTER(ctypes.c_int32)
_c_u16p = ctypes.POINTER(ctypes.c_uint16)
_c_f64p = ctypes.POINTER(ctypes.c_double)
_c_u8p = ctypes.POINTER(ctypes.c_uint8)
_c_f32p = ctypes.POINTER(ctypes.c_float)


def library_path(mutant: int = 0) -> Path:
    return HERE / ("liboracle.so" if mutant == 0 else f"liboracle_mutant{mutant}.so")


def build(mutant: int = 0, force: bool = False) -> Path:
    """Compile the oracle (optionally a planted-mistake variant); return the .so path."""
    out = library_path(mutant)
    if force or not out.exists() or out.stat().st_mtime < SRC.stat().st_mtime:
        tmp = out.with_suffix(f".so.tmp{os.getpid()}")
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-Wall", "-Wextra",
               f"-DORACLE_MUTANT={mutant}", "-o", str(tmp), str(SRC), "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, out)
    return out


class Oracle:
    """One loaded oracle library (the default build, or a planted-mistake variant)."""

    def __init__(self, mutant: int = 0):
        self.mutant = mutant
        self.lib = ctypes.CDLL(str(build(mutant)))
        L = self.lib
        i32, i64, f64, ci = ctypes.c_int32, ctypes.c_int64, ctypes.c_double, ctypes.c_int
        L.oracle_bf16_round.argtypes = [_c_f64p, _c_u16p, i64]
        L.oracle_kv_location.argtypes = [_c_i32p, i32, i32, i32, i32, i32, _c_i32p, _c_i32p]
        L.oracle_store_kvcache.argtypes = [_c_u16p, _c_u16p, i64, i64, _c_u16p, _c_u16p, _c_i32p, i32, i32, i32,
                                           i32, i32]
        L.oracle_decode.argtypes = [_c_u16p, _c_f64p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, i32, _c_i32p, i32, i32,
                                    i32, i32, i32, i32, f64, ci]
        L.oracle_decode_partials.argtypes = [_c_f64p, _c_f64p, _c_f64p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, i32,
                                             _c_i32p, i32, i32, i32, i32, i32, i32, f64, i32, i32]
        L.oracle_merge_partials.argtypes = [_c_u16p, _c_f64p, _c_f64p, _c_f64p, _c_f64p, i32, i32, i32]
        L.oracle_prefill_varlen.argtypes = [_c_u16p, _c_f64p, _c_u16p, _c_u16p, _c_u16p, _c_i32p, _c_i32p,
                                            _c_i32p, i32, i32, i32, i32, i32, i32, i32, f64, i32, _c_u8p, ci]
        L.oracle_rope_table.argtypes = [_c_f32p, i32, i32, f64]
        L.oracle_rope_store_kvcache.argtypes = [_c_u16p, _c_f64p, _c_u16p, i64, _c_u16p, _c_u16p, i64, i64, _c_i32p,
                                                _c_f32p, i32, _c_u16p, _c_u16p, _c_i32p, i32, i32, i32, i32, i32, i32]
        for name in ("oracle_bf16_round", "oracle_kv_location", "oracle_store_kvcache", "oracle_decode",
                     "oracle_decode_partials", "oracle_merge_partials", "oracle_prefill_varlen",
                     "oracle_rope_table", "oracle_rope_store_kvcache", "oracle_mutant_id", "oracle_max_threads"):
            getattr(L, name).restype = ctypes.c_int
        assert L.oracle_mutant_id() == mutant

    # -- helpers -------------------------------------------------------------------------------
    @staticmethod
    def _p(a, ct):
        return None if a is None else a.ctypes.data_as(ct)

    @staticmethod
    def _check(rc, what):
        if rc != 0:
            raise ValueError(f"oracle {what} failed with code {rc}")

    def max_threads(self) -> int:
        return int(self.lib.oracle_max_threads())

    # -- entry points --------------------------------------------------------------------------
    def bf16_round(self, x) -> np.ndarray:
        x = np.ascontiguousarray(x, dtype=np.float64)
        out = np.empty(x.shape, dtype=np.uint16)
        self._check(self.lib.oracle_bf16_round(self._p(x, _c_f64p), self._p(out, _c_u16p), x.size), "bf16_round")
        return out

    def kv_location(self, block_tables, b, pos, block_size, num_blocks):
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        blk, off = ctypes.c_int32(), ctypes.c_int32()
        self._check(self.lib.oracle_kv_location(self._p(bt, _c_i32p), bt.shape[1], b, pos, block_size, num_blocks,
                                                ctypes.byref(blk), ctypes.byref(off)), "kv_location")
        return blk.value, off.value

    def store_kvcache(self, key, value, k_cache, v_cache, slot_mapping):
        """In-place scatter of key/value rows ([N, Hkv, D] bf16 bits, row stride may exceed Hkv*D)."""
        assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
        nb, bs, hkv, d = k_cache.shape
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
        n = sm.shape[0]
        key2 = key.reshape(n, -1) if n else key.reshape(0, hkv * d)
        val2 = value.reshape(n, -1) if n else value.reshape(0, hkv * d)
        ks = key2.strides[0] // 2 if n else hkv * d
        vs = val2.strides[0] // 2 if n else hkv * d
        assert key2.strides[-1] == 2 and val2.strides[-1] == 2
        self._check(self.lib.oracle_store_kvcache(self._p(key2, _c_u16p), self._p(val2, _c_u16p), ks, vs,
                                                  self._p(k_cache, _c_u16p), self._p(v_cache, _c_u16p),
                                                  self._p(sm, _c_i32p), n, hkv, d, bs, nb), "store_kvcache")

    def rope_table(self, max_position, head_dim, base):
        """Rotary cos/sin cache [max_position, head_dim] float32: cos(p theta_i) then sin(p theta_i)."""
        t = np.empty((max_position, head_dim), dtype=np.float32)
        self._check(self.lib.oracle_rope_table(self._p(t, _c_f32p), max_position, head_dim, float(base)), "rope_table")
        return t

    def rope_store_kvcache(self, q, key, value, positions, table, k_cache, v_cache, slot_mapping, *, want_f64=False):
        """Rotate q ([N, Hq, D], row stride may exceed Hq*D) and key to their positions; store the rotated key
        and the value rows into the cache (slot -1 skipped).  Returns q_out [N, Hq, D] (and its doubles)."""
        assert k_cache.flags.c_contiguous and v_cache.flags.c_contiguous
        nb, bs, hkv, d = k_cache.shape
        n = int(np.asarray(positions).shape[0])
        hq = q.shape[1]
        pos = np.ascontiguousarray(positions, dtype=np.int32)
        sm = np.ascontiguousarray(slot_mapping, dtype=np.int32)
        tab = np.ascontiguousarray(table, dtype=np.float32)
        rows = []
        for a, h in ((q, hq), (key, hkv), (value, hkv)):
            a2 = a.reshape(n, -1) if n else np.zeros((0, h * d), np.uint16)
            assert a2.strides[-1] == 2
            rows.append((a2, a2.strides[0] // 2 if n else h * d))
        out = np.zeros((n, hq, d), dtype=np.uint16)
        of = np.zeros((n, hq, d), dtype=np.float64) if want_f64 else None
        (q2, qs), (k2, ks), (v2, vs) = rows
        self._check(self.lib.oracle_rope_store_kvcache(
            self._p(out, _c_u16p), self._p(of, _c_f64p), self._p(q2, _c_u16p), qs, self._p(k2, _c_u16p),
            self._p(v2, _c_u16p), ks, vs, self._p(pos, _c_i32p), self._p(tab, _c_f32p), tab.shape[0],
            self._p(k_cache, _c_u16p), self._p(v_cache, _c_u16p), self._p(sm, _c_i32p), n, hq, hkv, d, bs, nb),
            "rope_store_kvcache")
        return (out, of) if want_f64 else out

    def decode(self, q, k_cache, v_cache, block_tables, context_lens, scale, *, want_f64=False, nthreads=0):
        q = np.ascontiguousarray(q, dtype=np.uint16)
        B, H, D = q.shape
        nb, bs, hkv, d2 = k_cache.shape
        assert d2 == D
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        out = np.empty((B, H, D), dtype=np.uint16)
        of = np.empty((B, H, D), dtype=np.float64) if want_f64 else None
        self._check(self.lib.oracle_decode(self._p(out, _c_u16p), self._p(of, _c_f64p), self._p(q, _c_u16p),
                                           self._p(k_cache, _c_u16p), self._p(v_cache, _c_u16p),
                                           self._p(bt, _c_i32p), bt.shape[1], self._p(cl, _c_i32p), B, H, hkv, D,
                                           bs, nb, float(scale), nthreads), "decode")
        return (out, of) if want_f64 else out

    def decode_partials(self, q, k_cache, v_cache, block_tables, context_lens, scale, chunk_len, num_chunks):
        q = np.ascontiguousarray(q, dtype=np.uint16)
        B, H, D = q.shape
        nb, bs, hkv, _ = k_cache.shape
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        cl = np.ascontiguousarray(context_lens, dtype=np.int32)
        m = np.empty((B, H, num_chunks)); l = np.empty((B, H, num_chunks)); acc = np.empty((B, H, num_chunks, D))
        self._check(self.lib.oracle_decode_partials(self._p(m, _c_f64p), self._p(l, _c_f64p), self._p(acc, _c_f64p),
                                                    self._p(q, _c_u16p), self._p(k_cache, _c_u16p),
                                                    self._p(v_cache, _c_u16p), self._p(bt, _c_i32p), bt.shape[1],
                                                    self._p(cl, _c_i32p), B, H, hkv, D, bs, nb, float(scale),
                                                    chunk_len, num_chunks), "decode_partials")
        return m, l, acc

    def merge_partials(self, m, l, acc):
        m = np.ascontiguousarray(m, dtype=np.float64); l = np.ascontiguousarray(l, dtype=np.float64)
        acc = np.ascontiguousarray(acc, dtype=np.float64)
        *lead, C, D = acc.shape
        rows = int(np.prod(lead))
        out = np.empty((*lead, D), dtype=np.uint16)
        of = np.empty((*lead, D), dtype=np.float64)
        self._check(self.lib.oracle_merge_partials(self._p(out, _c_u16p), self._p(of, _c_f64p), self._p(m, _c_f64p),
                                                   self._p(l, _c_f64p), self._p(acc, _c_f64p), rows, C, D),
                    "merge_partials")
        return out, of

    def prefill_varlen(self, q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, block_tables, scale, causal=True,
                       *, row_select=None, want_f64=False, nthreads=0):
        q = np.ascontiguousarray(q, dtype=np.uint16)
        T, H, D = q.shape
        nb, bs, hkv, _ = k_cache.shape
        cq = np.ascontiguousarray(cu_seqlens_q, dtype=np.int32)
        ck = np.ascontiguousarray(cu_seqlens_k, dtype=np.int32)
        bt = np.ascontiguousarray(block_tables, dtype=np.int32)
        rs = None if row_select is None else np.ascontiguousarray(row_select, dtype=np.uint8)
        out = np.zeros((T, H, D), dtype=np.uint16)
        of = np.zeros((T, H, D), dtype=np.float64) if want_f64 else None
        self._check(self.lib.oracle_prefill_varlen(self._p(out, _c_u16p), self._p(of, _c_f64p), self._p(q, _c_u16p),
                                                   self._p(k_cache, _c_u16p), self._p(v_cache, _c_u16p),
                                                   self._p(cq, _c_i32p), self._p(ck, _c_i32p), self._p(bt, _c_i32p),
                                                   bt.shape[1], cq.shape[0] - 1, H, hkv, D, bs, nb, float(scale),
                                                   int(bool(causal)), self._p(rs, _c_u8p), nthreads),
                    "prefill_varlen")
        return (out, of) if want_f64 else out


_DEFAULT = None


def get() -> Oracle:
    """The default (mistake-free) oracle, loaded once."""
    global _DEFAULT
    if _DEFAULT is None:
        _DEFAULT = Oracle(0)
    return _DEFAULT
