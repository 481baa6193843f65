"""ctypes binding of libpagedattn.so (the C ABI declared in include/pa.h).

Argument marshalling only: torch tensors supply device pointers, shapes and
the current CUDA stream; every step of the computation runs in the library's
kernels.  There is no fallback: if the library is missing or the tensors are
not CUDA tensors, the call raises.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

LIB_PATH = Path(__file__).resolve().parent / "libpagedattn.so"

PA_OK = 0
_lib = None

_i32, _i64, _f32, _sz, _vp = ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t, ctypes.c_void_p

_PROTOS = {
    "pa_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "pa_last_error": (ctypes.c_char_p, []),
    "pa_version": (_i32, []),
    "pa_store_kvcache": (ctypes.c_int, [_vp, _vp, _i64, _i64, _vp, _vp, _vp, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pa_decode_chunk_size": (_i32, [_i32, _i32, _i32, _i32]),
    "pa_decode_chunk_size_for": (_i32, [_i32, _i32, _i32, _i32]),
    "pa_decode_workspace_size": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32, _i32]),
    "pa_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32, _f32,
                                 _i32, _vp, _sz, _vp]),
    "pa_prefill_varlen": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _i32, _i32, _vp, _i32, _i32, _i32, _i32,
                                         _i32, _i32, _i32, _f32, _i32, _vp]),
    "pa_device_error": (ctypes.c_int, [ctypes.POINTER(_i32), _vp]),
    "pa_decode_partial": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32,
                                         _i32, _i32, _f32, _i32, _vp, _sz, _vp]),
    "pa_merge_partials": (ctypes.c_int, [_vp, _vp, _vp, _i32, _i32, _i32, _vp]),
    "pa_store_decode": (ctypes.c_int, [_vp, _vp, _vp, _vp, _i64, _i64, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32,
                                       _i32, _i32, _i32, _i32, _f32, _i32, _vp, _sz, _vp]),
    "pa_rotary_cos_sin_cache": (ctypes.c_int, [_vp, _i32, _i32, ctypes.c_double, _vp]),
    "pa_rotary_store_kvcache": (ctypes.c_int, [_vp, _vp, _i64, _vp, _vp, _i64, _i64, _vp, _vp, _i32, _vp, _vp, _vp,
                                               _i32, _i32, _i32, _i32, _i32, _i32, _vp]),
    "pa_decode_noalloc": (ctypes.c_int, [_vp, _vp, _vp, _vp, _vp, _i32, _vp, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                         _f32, _i32, _vp]),
    "pa_selftest_wait_timeout": (ctypes.c_int, [_i64, _vp]),
}


class PagedAttentionError(RuntimeError):
    pass


def lib() -> ctypes.CDLL:
    """Load libpagedattn.so once; raise if it has not been built."""
    global _lib
    if _lib is None:
        if not LIB_PATH.exists():
            raise ImportError(f"{LIB_PATH.name} is missing; build it with `python -m paged_kv_cache_331_b200.build`")
        L = ctypes.CDLL(str(LIB_PATH))
        for name, (res, args) in _PROTOS.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _check(status: int, what: str) -> None:
    if status != PA_OK:
        L = lib()
        raise PagedAttentionError(f"{what}: {L.pa_status_string(status).decode()}: {L.pa_last_error().decode()}")


def _cuda(t: torch.Tensor, name: str, dtype=None) -> None:
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _dense(t: torch.Tensor, name: str) -> None:
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


def _same_device(ref: torch.Tensor, **tensors) -> None:
    """Every tensor of one call lives on the device of ``ref``: a pointer into
    another GPU's memory would reach a kernel that cannot read it."""
    for name, t in tensors.items():
        if t is not None and t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, the call's other tensors on {ref.device}")


def _shape(t: torch.Tensor, shape, name: str) -> None:
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")


def _rows(t: torch.Tensor, n: int, name: str, dim: int) -> None:
    """A per-sequence array (``dim`` dimensions) with at least one row per sequence; rows past n are not read."""
    if t.dim() != dim or t.shape[0] < n:
        raise ValueError(f"{name} must be {dim}-D with at least {n} rows, got shape {tuple(t.shape)}")


def _caches(k_cache: torch.Tensor, v_cache: torch.Tensor, head_dim=None) -> None:
    if k_cache.dim() != 4 or tuple(v_cache.shape) != tuple(k_cache.shape):
        raise ValueError("k_cache and v_cache must both be [num_blocks, block_size, num_kv_heads, head_dim]")
    if head_dim is not None and k_cache.shape[3] != head_dim:
        raise ValueError(f"head_dim of the cache ({k_cache.shape[3]}) and of q ({head_dim}) differ")


def _stream(t: torch.Tensor, stream) -> int:
    s = stream if stream is not None else torch.cuda.current_stream(t.device)
    return s.cuda_stream


def store_kvcache(key, value, k_cache, v_cache, slot_mapping, stream=None) -> None:
    """Scatter key/value rows [N, Hkv, D] into k_cache/v_cache at slot_mapping (-1 = skip)."""
    for n, t in (("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16)
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    _dense(k_cache, "k_cache"); _dense(v_cache, "v_cache"); _dense(slot_mapping, "slot_mapping")
    _caches(k_cache, v_cache)
    _same_device(k_cache, key=key, value=value, v_cache=v_cache, slot_mapping=slot_mapping)
    if slot_mapping.dim() != 1:
        raise ValueError("slot_mapping must be [N]")
    nb, bs, hkv, d = k_cache.shape
    n = slot_mapping.shape[0]
    for name, t in (("key", key), ("value", value)):
        if t.shape[0] != n or tuple(t.shape[1:]) != (hkv, d) or t.stride(-1) != 1 or t.stride(-2) != d:
            raise ValueError(f"{name} must be [N, {hkv}, {d}] with dense rows")
    with torch.cuda.device(k_cache.device):
        _check(lib().pa_store_kvcache(key.data_ptr(), value.data_ptr(), key.stride(0), value.stride(0),
                                      k_cache.data_ptr(), v_cache.data_ptr(), slot_mapping.data_ptr(), n, hkv, d, bs,
                                      nb, _stream(k_cache, stream)), "pa_store_kvcache")


def rotary_cos_sin_cache(max_position, head_dim, base, device=None, stream=None) -> torch.Tensor:
    """pa_rotary_cos_sin_cache: a new [max_position, head_dim] float32 table, cos(p theta_i) | sin(p theta_i)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    table = torch.empty(max_position, head_dim, dtype=torch.float32, device=dev)
    with torch.cuda.device(dev):
        _check(lib().pa_rotary_cos_sin_cache(table.data_ptr(), max_position, head_dim, float(base),
                                             _stream(table, stream)), "pa_rotary_cos_sin_cache")
    return table


def rotary_store_kvcache(q, key, value, positions, cos_sin_cache, k_cache, v_cache, slot_mapping, *, out=None,
                         stream=None) -> torch.Tensor:
    """pa_rotary_store_kvcache: rotate q [N, Hq, D] and key [N, Hkv, D] to their positions, store the rotated key and
    the value into the cache at slot_mapping (-1 = skip); returns the rotated q ([N, Hq, D], dense; ``out`` may be
    q itself when q is dense)."""
    for n, t in (("q", q), ("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16)
    _cuda(positions, "positions", torch.int32)
    _cuda(slot_mapping, "slot_mapping", torch.int32)
    _cuda(cos_sin_cache, "cos_sin_cache", torch.float32)
    for n, t in (("k_cache", k_cache), ("v_cache", v_cache), ("positions", positions), ("slot_mapping", slot_mapping),
                 ("cos_sin_cache", cos_sin_cache)):
        _dense(t, n)
    _caches(k_cache, v_cache)
    nb, bs, hkv, d = k_cache.shape
    if q.dim() != 3:
        raise ValueError("q must be [N, Hq, D]")
    n, hq = q.shape[0], q.shape[1]
    if tuple(q.shape[1:]) != (hq, d) or q.stride(-1) != 1 or q.stride(-2) != d:
        raise ValueError(f"q must be [N, Hq, {d}] with dense rows")
    for name, t in (("key", key), ("value", value)):
        if t.shape[0] != n or tuple(t.shape[1:]) != (hkv, d) or t.stride(-1) != 1 or t.stride(-2) != d:
            raise ValueError(f"{name} must be [N, {hkv}, {d}] with dense rows")
    if positions.shape != (n,) or slot_mapping.shape != (n,):
        raise ValueError("positions and slot_mapping must be [N]")
    if cos_sin_cache.dim() != 2 or cos_sin_cache.shape[1] != d:
        raise ValueError(f"cos_sin_cache must be [max_position, {d}]")
    if out is None:
        out = torch.empty(n, hq, d, dtype=torch.bfloat16, device=q.device)
    _cuda(out, "out", torch.bfloat16)
    _dense(out, "out")
    _shape(out, (n, hq, d), "out")
    _same_device(k_cache, q=q, key=key, value=value, positions=positions, cos_sin_cache=cos_sin_cache,
                 v_cache=v_cache, slot_mapping=slot_mapping, out=out)
    with torch.cuda.device(k_cache.device):
        _check(lib().pa_rotary_store_kvcache(out.data_ptr(), q.data_ptr(), q.stride(0), key.data_ptr(),
                                             value.data_ptr(), key.stride(0), value.stride(0), positions.data_ptr(),
                                             cos_sin_cache.data_ptr(), cos_sin_cache.shape[0], k_cache.data_ptr(),
                                             v_cache.data_ptr(), slot_mapping.data_ptr(), n, hq, hkv, d, bs, nb,
                                             _stream(k_cache, stream)), "pa_rotary_store_kvcache")
    return out


def decode_chunk_size(num_seqs, num_kv_heads, max_context_len, block_size) -> int:
    return int(lib().pa_decode_chunk_size(num_seqs, num_kv_heads, max_context_len, block_size))


def decode_chunk_size_for(num_seqs, num_kv_heads, max_context_len, sm_count) -> int:
    return int(lib().pa_decode_chunk_size_for(num_seqs, num_kv_heads, max_context_len, sm_count))


def decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len, block_size,
                          kv_chunk_size=0) -> int:
    return int(lib().pa_decode_workspace_size(num_seqs, num_heads, num_kv_heads, head_dim, max_context_len,
                                              block_size, kv_chunk_size))


def decode(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, *, out=None, workspace=None,
           kv_chunk_size=0, stream=None):
    """Paged GQA decode: q [B, Hq, D] -> out [B, Hq, D]."""
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16); _dense(t, n)
    _cuda(block_tables, "block_tables", torch.int32); _dense(block_tables, "block_tables")
    _cuda(context_lens, "context_lens", torch.int32); _dense(context_lens, "context_lens")
    B, hq, d = q.shape
    _caches(k_cache, v_cache, d)
    nb, bs, hkv, _ = k_cache.shape
    _rows(block_tables, B, "block_tables", 2)
    _rows(context_lens, B, "context_lens", 1)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out, "out", torch.bfloat16); _dense(out, "out"); _shape(out, q.shape, "out")
    need = decode_workspace_size(B, hq, hkv, d, int(max_context_len), bs, kv_chunk_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _same_device(q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables, context_lens=context_lens, out=out,
                 workspace=workspace)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(q.device):
        _check(lib().pa_decode(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                               block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
                               int(max_context_len), B, hq, hkv, d, bs, nb, float(scale), int(kv_chunk_size), ws_ptr,
                               ws_len, _stream(q, stream)), "pa_decode")
    return out


def store_decode(q, key, value, slot_mapping, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, *,
                 out=None, workspace=None, kv_chunk_size=0, stream=None, validate=False):
    """pa_store_decode: store each sequence's new K/V row (slot of position L-1, or -1) and decode, one launch.

    ``validate=True`` first checks on the host (a synchronising copy) that every slot is the one its block table
    names for the newest position, through a valid block id, and raises before the launch.  Without it the kernel
    still skips a slot that breaks this and records device error code 5 or 6 (read with ``device_error()``)."""
    for n, t in (("q", q), ("key", key), ("value", value), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16)
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _dense(t, n)
    for n, t in (("slot_mapping", slot_mapping), ("block_tables", block_tables), ("context_lens", context_lens)):
        _cuda(t, n, torch.int32)
        _dense(t, n)
    B, hq, d = q.shape
    _caches(k_cache, v_cache, d)
    nb, bs, hkv, _ = k_cache.shape
    for name, t in (("key", key), ("value", value)):
        if t.shape[0] != B or tuple(t.shape[1:]) != (hkv, d) or t.stride(-1) != 1 or t.stride(-2) != d:
            raise ValueError(f"{name} must be [B, {hkv}, {d}] with dense rows")
    _rows(slot_mapping, B, "slot_mapping", 1)
    _rows(block_tables, B, "block_tables", 2)
    _rows(context_lens, B, "context_lens", 1)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out, "out", torch.bfloat16); _dense(out, "out"); _shape(out, q.shape, "out")
    need = decode_workspace_size(B, hq, hkv, d, int(max_context_len), bs, kv_chunk_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _same_device(q, key=key, value=value, slot_mapping=slot_mapping, k_cache=k_cache, v_cache=v_cache,
                 block_tables=block_tables, context_lens=context_lens, out=out, workspace=workspace)
    if validate:
        from .metadata import check_store_decode_metadata
        check_store_decode_metadata(slot_mapping[:B], block_tables[:B], context_lens[:B], int(max_context_len), bs, nb)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(q.device):
        _check(lib().pa_store_decode(out.data_ptr(), q.data_ptr(), key.data_ptr(), value.data_ptr(), key.stride(0),
                                     value.stride(0), slot_mapping.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                     block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
                                     int(max_context_len), B, hq, hkv, d, bs, nb, float(scale), kv_chunk_size, ws_ptr,
                                     ws_len, _stream(q, stream)), "pa_store_decode")
    return out


def decode_partial(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, *, o_part=None,
                   lse_part=None, workspace=None, kv_chunk_size=0, stream=None):
    """pa_decode_partial: fp32 partial (o [B, Hq, D], lse [B, Hq] in log2 units) over the keys the tables name."""
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16)
        _dense(t, n)
    _cuda(block_tables, "block_tables", torch.int32)
    _cuda(context_lens, "context_lens", torch.int32)
    _dense(block_tables, "block_tables")
    _dense(context_lens, "context_lens")
    B, hq, d = q.shape
    _caches(k_cache, v_cache, d)
    nb, bs, hkv, _ = k_cache.shape
    _rows(block_tables, B, "block_tables", 2)
    _rows(context_lens, B, "context_lens", 1)
    if o_part is None:
        o_part = torch.empty(B, hq, d, dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty(B, hq, dtype=torch.float32, device=q.device)
    for n, t in (("o_part", o_part), ("lse_part", lse_part)):
        _cuda(t, n, torch.float32)
        _dense(t, n)
    _shape(o_part, (B, hq, d), "o_part")
    _shape(lse_part, (B, hq), "lse_part")
    need = decode_workspace_size(B, hq, hkv, d, int(max_context_len), bs, kv_chunk_size)
    if need and workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=q.device)
    _same_device(q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables, context_lens=context_lens,
                 o_part=o_part, lse_part=lse_part, workspace=workspace)
    ws_ptr = workspace.data_ptr() if workspace is not None else None
    ws_len = workspace.numel() * workspace.element_size() if workspace is not None else 0
    with torch.cuda.device(q.device):
        _check(lib().pa_decode_partial(o_part.data_ptr(), lse_part.data_ptr(), q.data_ptr(), k_cache.data_ptr(),
                                       v_cache.data_ptr(), block_tables.data_ptr(), block_tables.shape[1],
                                       context_lens.data_ptr(), int(max_context_len), B, hq, hkv, d, bs, nb,
                                       float(scale), kv_chunk_size, ws_ptr, ws_len, _stream(q, stream)),
               "pa_decode_partial")
    return o_part, lse_part


def merge_partials(o_parts, lse_parts, *, out=None, stream=None):
    """pa_merge_partials: o_parts [R, B, Hq, D] fp32 and lse_parts [R, B, Hq] fp32 -> out [B, Hq, D] bf16."""
    _cuda(o_parts, "o_parts", torch.float32)
    _cuda(lse_parts, "lse_parts", torch.float32)
    _dense(o_parts, "o_parts")
    _dense(lse_parts, "lse_parts")
    if o_parts.dim() != 4:
        raise ValueError("o_parts must be [R, B, Hq, D]")
    R, B, hq, d = o_parts.shape
    if tuple(lse_parts.shape) != (R, B, hq):
        raise ValueError("lse_parts must be [R, B, Hq]")
    if out is None:
        out = torch.empty(B, hq, d, dtype=torch.bfloat16, device=o_parts.device)
    _cuda(out, "out", torch.bfloat16)
    _dense(out, "out")
    _shape(out, (B, hq, d), "out")
    _same_device(o_parts, lse_parts=lse_parts, out=out)
    with torch.cuda.device(o_parts.device):
        _check(lib().pa_merge_partials(out.data_ptr(), o_parts.data_ptr(), lse_parts.data_ptr(), R, B * hq, d,
                                       _stream(o_parts, stream)), "pa_merge_partials")
    return out


def decode_noalloc(q, k_cache, v_cache, block_tables, context_lens, max_context_len, scale, *, out, kv_chunk_size=0,
                   stream=None):
    """pa_decode_noalloc: decode with the library's fixed split-KV scratch (no workspace, nothing allocated).

    For callers that cannot provide device memory of their own; ``out`` must be given.  Calls that may run
    concurrently on one GPU share the scratch and must be ordered."""
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache), ("out", out)):
        _cuda(t, n, torch.bfloat16); _dense(t, n)
    _cuda(block_tables, "block_tables", torch.int32); _dense(block_tables, "block_tables")
    _cuda(context_lens, "context_lens", torch.int32); _dense(context_lens, "context_lens")
    B, hq, d = q.shape
    _caches(k_cache, v_cache, d)
    nb, bs, hkv, _ = k_cache.shape
    _rows(block_tables, B, "block_tables", 2)
    _rows(context_lens, B, "context_lens", 1)
    _shape(out, q.shape, "out")
    _same_device(q, k_cache=k_cache, v_cache=v_cache, block_tables=block_tables, context_lens=context_lens, out=out)
    with torch.cuda.device(q.device):
        _check(lib().pa_decode_noalloc(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                       block_tables.data_ptr(), block_tables.shape[1], context_lens.data_ptr(),
                                       int(max_context_len), B, hq, hkv, d, bs, nb, float(scale), int(kv_chunk_size),
                                       _stream(q, stream)), "pa_decode_noalloc")
    return out


def prefill_varlen(q, k_cache, v_cache, cu_seqlens_q, cu_seqlens_k, max_seqlen_q, max_seqlen_k, block_tables, scale,
                   causal=True, *, out=None, stream=None, validate=False):
    """Varlen prefill over the paged cache: q [total_q, Hq, D] -> out [total_q, Hq, D].

    ``validate=True`` first checks on the host (a synchronising copy) that the cu_seqlens agree with total_q,
    max_seqlen_q/k and the block tables, whose entries are valid block ids, and raises before the launch.  Without
    it the kernel still skips a sequence whose metadata breaks this (device error code 8) and reads zeros for a
    block id outside the cache (code 6)."""
    for n, t in (("q", q), ("k_cache", k_cache), ("v_cache", v_cache)):
        _cuda(t, n, torch.bfloat16); _dense(t, n)
    for n, t in (("cu_seqlens_q", cu_seqlens_q), ("cu_seqlens_k", cu_seqlens_k), ("block_tables", block_tables)):
        _cuda(t, n, torch.int32); _dense(t, n)
    total_q, hq, d = q.shape
    _caches(k_cache, v_cache, d)
    nb, bs, hkv, _ = k_cache.shape
    if cu_seqlens_q.dim() != 1 or cu_seqlens_q.shape[0] < 1:
        raise ValueError("cu_seqlens_q must be [num_seqs + 1]")
    num_seqs = cu_seqlens_q.shape[0] - 1
    _rows(cu_seqlens_k, num_seqs + 1, "cu_seqlens_k", 1)
    _rows(block_tables, num_seqs, "block_tables", 2)
    if out is None:
        out = torch.empty_like(q)
    else:
        _cuda(out, "out", torch.bfloat16); _dense(out, "out"); _shape(out, q.shape, "out")
    _same_device(q, k_cache=k_cache, v_cache=v_cache, cu_seqlens_q=cu_seqlens_q, cu_seqlens_k=cu_seqlens_k,
                 block_tables=block_tables, out=out)
    if validate:
        from .metadata import check_prefill_metadata
        check_prefill_metadata(cu_seqlens_q, cu_seqlens_k[:num_seqs + 1], total_q, int(max_seqlen_q),
                               int(max_seqlen_k), block_tables, bs, nb)
    with torch.cuda.device(q.device):
        _check(lib().pa_prefill_varlen(out.data_ptr(), q.data_ptr(), k_cache.data_ptr(), v_cache.data_ptr(),
                                       cu_seqlens_q.data_ptr(), cu_seqlens_k.data_ptr(), total_q, int(max_seqlen_q),
                                       int(max_seqlen_k), block_tables.data_ptr(), block_tables.shape[1],
                                       num_seqs, hq, hkv, d, bs, nb, float(scale), int(bool(causal)),
                                       _stream(q, stream)), "pa_prefill_varlen")
    return out


def device_error(stream=None, device=None) -> int:
    """Read and clear the library's device-side error word (synchronises the stream)."""
    dev = device if device is not None else torch.cuda.current_device()
    code = _i32(0)
    with torch.cuda.device(dev):
        s = stream.cuda_stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
        _check(lib().pa_device_error(ctypes.byref(code), s), "pa_device_error")
    return int(code.value)


def selftest_wait_timeout(limit_ns: int, stream=None, device=None) -> None:
    """Launch the one-CTA kernel whose pipeline wait has nothing to arrive on: it gives up after limit_ns,
    records code 1 (read it with device_error()), frees its tensor memory and returns."""
    dev = device if device is not None else torch.cuda.current_device()
    with torch.cuda.device(dev):
        s = stream.cuda_stream if stream is not None else torch.cuda.current_stream(dev).cuda_stream
        _check(lib().pa_selftest_wait_timeout(int(limit_ns), s), "pa_selftest_wait_timeout")
