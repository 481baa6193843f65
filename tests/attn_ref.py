"""Library-routine references used to pin the oracle (CPU, float64).

The attention math here is torch's own ``scaled_dot_product_attention`` and
its ``causal_lower_right`` bias; the only thing these helpers do by hand is
lay the paged cache out contiguously for one sequence, by numpy indexing of
the block table.
"""
import numpy as np
import torch
import torch.nn.functional as F
from torch.nn.attention.bias import causal_lower_right

from paged_kv_cache_331_b200.workloads import bf16_bits_to_f32


def gather_contiguous(cache, table, n, block_size):
    """[n, Hkv, D] float64 rows of logical positions 0..n-1 of one sequence."""
    pos = np.arange(n)
    rows = cache[table[pos // block_size], pos % block_size]
    return torch.from_numpy(bf16_bits_to_f32(rows).astype(np.float64))


def sdpa_rows(q_rows, k, v, scale, mask=None):
    """q_rows [Lq, Hq, D]; k, v [Lk, Hkv, D] float64 -> [Lq, Hq, D] via torch SDPA (GQA by head groups)."""
    hq, hkv = q_rows.shape[1], k.shape[1]
    qt = q_rows.permute(1, 0, 2).unsqueeze(0)                 # [1, Hq, Lq, D]
    kt = k.permute(1, 0, 2).unsqueeze(0)                      # [1, Hkv, Lk, D]
    vt = v.permute(1, 0, 2).unsqueeze(0)
    o = F.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask, scale=scale, enable_gqa=(hq != hkv))
    return o.squeeze(0).permute(1, 0, 2)


def decode_reference(w):
    """Float64 SDPA decode of a DecodeWorkload whose new rows are already in its caches."""
    out = np.zeros((w.num_seqs, w.num_heads, w.head_dim))
    for b in range(w.num_seqs):
        L = int(w.context_lens[b])
        if L == 0:
            continue
        k = gather_contiguous(w.k_cache, w.block_tables[b], L, w.block_size)
        v = gather_contiguous(w.v_cache, w.block_tables[b], L, w.block_size)
        q = torch.from_numpy(bf16_bits_to_f32(w.q[b:b + 1]).astype(np.float64))
        out[b] = sdpa_rows(q, k, v, w.scale)[0].numpy()
    return out


def prefill_reference(w):
    """Float64 SDPA prefill (bottom-right causal mask from torch when causal)."""
    T = int(w.cu_seqlens_q[-1])
    out = np.zeros((T, w.num_heads, w.head_dim))
    for b in range(w.num_seqs):
        q0, q1 = int(w.cu_seqlens_q[b]), int(w.cu_seqlens_q[b + 1])
        Lq, Lk = q1 - q0, int(w.cu_seqlens_k[b + 1] - w.cu_seqlens_k[b])
        if Lq == 0:
            continue
        k = gather_contiguous(w.k_cache, w.block_tables[b], Lk, w.block_size)
        v = gather_contiguous(w.v_cache, w.block_tables[b], Lk, w.block_size)
        q = torch.from_numpy(bf16_bits_to_f32(w.q[q0:q1]).astype(np.float64))
        mask = causal_lower_right(Lq, Lk) if w.causal else None
        out[q0:q1] = sdpa_rows(q, k, v, w.scale, mask).numpy()
    return out
