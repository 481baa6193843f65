"""GPU parity of the rotary embedding entry points against the oracle.

Tolerance, from the arithmetic: the kernel forms x_i cos - x_{i+D/2} sin (and the
partner) in float with one rounded product and one fused multiply-add, then rounds
to bf16; the oracle forms it exactly in double and rounds once.  Before the final
rounding the two differ by at most 2^-23 (|x_i| + |x_{i+D/2}|) (|cos|, |sin| <= 1),
and a bf16 rounding adds at most half a bf16 ulp <= 2^-9 |y|.  So every element
obeys |gpu - exact| <= 2^-8 |exact| + 2^-22 (|x_i| + |x_{i+D/2}|), and elements away
from a rounding boundary are bit-equal to the oracle's bf16.
"""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import dev_bf16, dev_i32, host_bits

pytestmark = pytest.mark.gpu


def _f(bits):
    return (np.asarray(bits).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def _check_rotated(gpu_bits, ref_bits, ref_f64, x_bits, what):
    d = x_bits.shape[-1]
    xf = _f(x_bits)
    pair = np.abs(xf[..., : d // 2]) + np.abs(xf[..., d // 2:])
    pair = np.concatenate([pair, pair], axis=-1)
    err = np.abs(_f(gpu_bits) - ref_f64)
    bound = 2.0 ** -8 * np.abs(ref_f64) + 2.0 ** -22 * pair
    assert (err <= bound).all(), f"{what}: {int((err > bound).sum())} elements outside the bound"
    same = (gpu_bits == ref_bits).mean()
    assert same >= 0.999, f"{what}: only {same:.5f} of elements bit-equal to the oracle"


@pytest.mark.parametrize("d,base,maxpos", [(128, 1e6, 40960), (64, 1e4, 4096)])
def test_cos_sin_cache_matches_oracle(oracle, d, base, maxpos):
    t = pa.rotary_cos_sin_cache(maxpos, d, base, device="cuda").cpu().numpy()
    ref = oracle.rope_table(maxpos, d, base)
    ulps = np.abs(t.view(np.int32).astype(np.int64) - ref.view(np.int32).astype(np.int64))
    assert ulps.max() <= 1
    assert (ulps == 0).mean() > 0.9999


CASES = [  # tokens, Hq, Hkv, D, block_size, fused QKV view
    (7, 8, 2, 128, 16, True),
    (300, 16, 8, 128, 256, True),
    (65, 4, 4, 64, 32, False),
    (1, 32, 8, 128, 256, False),
    (129, 6, 1, 64, 16, True),
]


@pytest.mark.parametrize("n,hq,hkv,d,bs,fused", CASES)
def test_rotary_store_matches_oracle(oracle, n, hq, hkv, d, bs, fused):
    rng = np.random.default_rng(1000 + n + hq)
    maxpos = 8192
    table = oracle.rope_table(maxpos, d, 1e6 if d == 128 else 1e4)
    nb = (n + bs - 1) // bs + 3
    if fused:
        qkv = W.randn_bf16(rng, (n, (hq + 2 * hkv) * d))
        q = qkv[:, : hq * d].reshape(n, hq, d)
        key = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d)
        val = qkv[:, (hq + hkv) * d:].reshape(n, hkv, d)
    else:
        qkv = None
        q, key, val = W.randn_bf16(rng, (n, hq, d)), W.randn_bf16(rng, (n, hkv, d)), W.randn_bf16(rng, (n, hkv, d))
    pos = rng.integers(0, maxpos, n).astype(np.int32)
    slots = rng.permutation(nb * bs)[:n].astype(np.int32)
    slots[rng.random(n) < 0.2] = -1
    kc = np.full((nb, bs, hkv, d), 0x7FC0, np.uint16)
    vc = kc.copy()
    kc_ref, vc_ref = kc.copy(), vc.copy()
    qo_ref, qo_f64 = oracle.rope_store_kvcache(q, key, val, pos, table, kc_ref, vc_ref, slots, want_f64=True)
    # rotated keys in double, for the bound on the K cache rows
    _, k_f64 = oracle.rope_store_kvcache(np.ascontiguousarray(key), key, key, pos, table,
                                         np.zeros((1, bs, hkv, d), np.uint16), np.zeros((1, bs, hkv, d), np.uint16),
                                         np.full(n, -1, np.int32), want_f64=True)

    if fused:
        dqkv = dev_bf16(qkv)
        dq = dqkv[:, : hq * d].view(n, hq, d)
        dk = dqkv[:, hq * d:(hq + hkv) * d].view(n, hkv, d)
        dv = dqkv[:, (hq + hkv) * d:].view(n, hkv, d)
    else:
        dq, dk, dv = dev_bf16(q), dev_bf16(key), dev_bf16(val)
    dkc, dvc = dev_bf16(kc), dev_bf16(vc)
    dtab = torch.from_numpy(table).cuda()
    qo = pa.rotary_store_kvcache(dq, dk, dv, dev_i32(pos), dtab, dkc, dvc, dev_i32(slots))
    torch.cuda.synchronize()
    assert pa.device_error() == 0
    _check_rotated(host_bits(qo), qo_ref, qo_f64, q, "q_out")
    live = slots >= 0
    kg = host_bits(dkc).reshape(-1, hkv, d)
    _check_rotated(kg[slots[live]], kc_ref.reshape(-1, hkv, d)[slots[live]], k_f64[live], key[live], "k_cache rows")
    # value rows bit-exact; every slot not written keeps its sentinel
    assert np.array_equal(host_bits(dvc), vc_ref)
    untouched = np.ones(nb * bs, bool)
    untouched[slots[live]] = False
    assert np.array_equal(kg[untouched], kc.reshape(-1, hkv, d)[untouched])


def test_rotary_store_in_place(oracle):
    rng = np.random.default_rng(77)
    n, hq, hkv, d, bs = 40, 8, 2, 128, 16
    table = oracle.rope_table(2048, d, 1e6)
    q, key, val = W.randn_bf16(rng, (n, hq, d)), W.randn_bf16(rng, (n, hkv, d)), W.randn_bf16(rng, (n, hkv, d))
    pos = rng.integers(0, 2048, n).astype(np.int32)
    slots = np.arange(n, dtype=np.int32)
    kc = np.zeros((4, bs, hkv, d), np.uint16)
    dtab = torch.from_numpy(table).cuda()
    dq = dev_bf16(q)
    dkc, dvc = dev_bf16(kc), dev_bf16(kc)
    ref = pa.rotary_store_kvcache(dev_bf16(q), dev_bf16(key), dev_bf16(val), dev_i32(pos), dtab, dkc.clone(),
                                  dvc.clone(), dev_i32(slots))
    got = pa.rotary_store_kvcache(dq, dev_bf16(key), dev_bf16(val), dev_i32(pos), dtab, dkc, dvc, dev_i32(slots),
                                  out=dq)
    torch.cuda.synchronize()
    assert got.data_ptr() == dq.data_ptr()
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_rotary_position_out_of_range_is_reported_not_written(oracle):
    d, hq, hkv, bs = 64, 2, 1, 16
    table = torch.from_numpy(oracle.rope_table(16, d, 1e4)).cuda()
    rng = np.random.default_rng(5)
    q, key, val = W.randn_bf16(rng, (3, hq, d)), W.randn_bf16(rng, (3, hkv, d)), W.randn_bf16(rng, (3, hkv, d))
    out = torch.zeros(3, hq, d, dtype=torch.bfloat16, device="cuda")
    kc = torch.zeros(1, bs, hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    pa.device_error()
    pa.rotary_store_kvcache(dev_bf16(q), dev_bf16(key), dev_bf16(val), dev_i32(np.array([3, 16, 5], np.int32)), table,
                            kc, vc, dev_i32(np.array([0, 1, 2], np.int32)), out=out)
    assert pa.device_error() == 4
    assert not out[1].any() and not kc[0, 1].any()          # the bad token's q and k rows are not written
    assert out[0].any() and kc[0, 0].any() and kc[0, 2].any()
    assert torch.equal(vc[0, 1].view(torch.int16).cpu(), torch.from_numpy(val[1].view(np.int16)))


def test_rotary_then_decode_matches_oracle_chain(oracle):
    """Decode step of a Qwen3-shaped layer: rotary store of the new token at position L-1, then decode."""
    from gpu_helpers import DeviceDecode, assert_attention_close
    rng = np.random.default_rng(31)
    lens = rng.integers(1, 3000, 24).astype(np.int32)
    w = W.decode_workload(lens, 16, 8, 128, 256, rng=rng)
    table = oracle.rope_table(4096, 128, 1e6)
    pos = (lens - 1).astype(np.int32)
    dw = DeviceDecode(w)
    qr = pa.rotary_store_kvcache(dw.q, dw.new_k, dw.new_v, dev_i32(pos), torch.from_numpy(table).cuda(), dw.k_cache,
                                 dw.v_cache, dw.slot_mapping)
    out = pa.decode(qr, dw.k_cache, dw.v_cache, dw.block_tables, dw.context_lens, int(lens.max()), w.scale)
    torch.cuda.synchronize()
    q_rot = oracle.rope_store_kvcache(w.q, w.new_k, w.new_v, pos, table, w.k_cache, w.v_cache, w.slot_mapping)
    _, ref = oracle.decode(q_rot, w.k_cache, w.v_cache, w.block_tables, w.context_lens, w.scale, want_f64=True)
    assert_attention_close(out, ref, what="rotary + decode")
    assert pa.device_error() == 0
