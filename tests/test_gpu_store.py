"""store_kvcache on the GPU, bit-exact against the oracle (whole caches compared)."""
import numpy as np
import pytest
import torch

import paged_kv_cache_331_b200 as pa
from paged_kv_cache_331_b200 import workloads as W
from gpu_helpers import DeviceDecode, DevicePrefill, dev_bf16, dev_i32, host_bits

pytestmark = pytest.mark.gpu


def run_both(oracle, key, value, k0, v0, slots, key_dev=None, value_dev=None):
    kc, vc = k0.copy(), v0.copy()
    oracle.store_kvcache(key, value, kc, vc, slots)
    kd, vd = dev_bf16(k0), dev_bf16(v0)
    pa.store_kvcache(key_dev if key_dev is not None else dev_bf16(key),
                     value_dev if value_dev is not None else dev_bf16(value), kd, vd, dev_i32(slots))
    torch.cuda.synchronize()
    assert np.array_equal(host_bits(kd), kc)
    assert np.array_equal(host_bits(vd), vc)


@pytest.mark.parametrize("hkv,d,bs", [(2, 64, 16), (8, 128, 256), (1, 128, 32), (4, 64, 1024)])
def test_store_random_slots_with_skips(oracle, hkv, d, bs):
    rng = np.random.default_rng(100 + d + bs)
    nb, n = 9, 300
    k0 = W.randn_bf16(rng, (nb, bs, hkv, d)); v0 = W.randn_bf16(rng, (nb, bs, hkv, d))
    n = min(n, nb * bs)
    slots = rng.choice(nb * bs, size=n, replace=False).astype(np.int32)
    slots[rng.random(n) < 0.2] = -1
    key = W.randn_bf16(rng, (n, hkv, d)); val = W.randn_bf16(rng, (n, hkv, d))
    run_both(oracle, key, val, k0, v0, slots)


def test_store_all_skipped_and_empty(oracle):
    rng = np.random.default_rng(5)
    k0 = W.randn_bf16(rng, (3, 16, 2, 64)); v0 = W.randn_bf16(rng, (3, 16, 2, 64))
    key = W.randn_bf16(rng, (7, 2, 64)); val = W.randn_bf16(rng, (7, 2, 64))
    run_both(oracle, key, val, k0, v0, np.full(7, -1, np.int32))
    run_both(oracle, key[:0], val[:0], k0, v0, np.zeros(0, np.int32))


@pytest.mark.parametrize("extra", [0, 4, 1])
def test_store_views_of_fused_qkv(oracle, extra):
    """key/value are strided views of a [N, (Hq + 2 Hkv) * D + extra] buffer; extra=1 and 4 force the
    narrow-access paths (rows not 16-byte aligned)."""
    rng = np.random.default_rng(6 + extra)
    hq, hkv, d, n = 4, 2, 64, 33
    width = (hq + 2 * hkv) * d + extra
    qkv = W.randn_bf16(rng, (n, width))
    key = qkv[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d)
    val = qkv[:, (hq + hkv) * d:(hq + 2 * hkv) * d].reshape(n, hkv, d)
    qkv_dev = dev_bf16(qkv)
    key_dev = qkv_dev[:, hq * d:(hq + hkv) * d].view(n, hkv, d)
    val_dev = qkv_dev[:, (hq + hkv) * d:(hq + 2 * hkv) * d].view(n, hkv, d)
    k0 = W.randn_bf16(rng, (4, 16, hkv, d)); v0 = W.randn_bf16(rng, (4, 16, hkv, d))
    slots = rng.permutation(64)[:n].astype(np.int32)
    run_both(oracle, key, val, k0, v0, slots, key_dev, val_dev)


@pytest.mark.parametrize("make", [W.tiny_decode, W.large_batch_decode])
def test_store_decode_workloads(oracle, make):
    w = make()
    run_both(oracle, w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)


def test_store_prefix_prefill_suffix_rows(oracle):
    """The ~9k suffix rows of the prefix-cached prefill workload, 4 shared prefix blocks untouched."""
    w = W.prefix_prefill()
    run_both(oracle, w.new_k, w.new_v, w.k_cache, w.v_cache, w.slot_mapping)
