"""The engine's attention steps end to end, on the GPU, against the oracle chain.

The C++ block manager plans every step, following "Architektur im Überblick"
(Block Manager, Hash-basiertes Prefix Caching, Dynamische Block-Erweiterung,
Prefill- und Decode-Vorbereitung):
- prefix-cache hits on a shared system prompt;
- prefill of only the uncached tokens;
- decode growth across block boundaries;
- release, then revival of freed prefix blocks whose K/V still sit in the cache.

The library executes each step: rotary store (q and k rotated to their positions,
k/v stored) followed by prefill or decode.  The oracle side replays the same
steps with the oracle block manager, the oracle rotary store and the oracle
attention.  The two plans must be identical and the attention outputs within
tolerance.

No model is involved.  A token's q/k/v are drawn from a generator seeded by the
token ids up to and including it, so sequences with equal prefixes produce
equal K/V, as a model would.
"""
import numpy as np
import pytest
import torch
import xxhash

import paged_kv_cache_331_b200 as pa
from oracle.block_manager import OracleBlockManager
from paged_kv_cache_331_b200 import workloads as W
from paged_kv_cache_331_b200.block_manager import BlockManager
from gpu_helpers import assert_attention_close, dev_bf16, dev_i32, host_bits

pytestmark = pytest.mark.gpu

HQ, HKV, D, BS, NBLK, MAXB = 8, 2, 128, 16, 48, 16
SCALE = 1.0 / np.sqrt(D)


def token_qkv(tokens_upto):
    rng = np.random.default_rng(xxhash.xxh64_intdigest(np.asarray(tokens_upto, np.int32).tobytes()))
    return W.randn_bf16(rng, (HQ, D)), W.randn_bf16(rng, (HKV, D)), W.randn_bf16(rng, (HKV, D))


class Flow:
    def __init__(self, oracle):
        self.oracle = oracle
        self.lib = BlockManager(NBLK, BS)
        self.orc = OracleBlockManager(NBLK, BS)
        self.table = oracle.rope_table(4096, D, 1e4)
        self.dtable = torch.from_numpy(self.table).cuda()
        self.kc = np.zeros((NBLK, BS, HKV, D), np.uint16)
        self.vc = np.zeros_like(self.kc)
        self.dkc, self.dvc = dev_bf16(self.kc), dev_bf16(self.vc)
        self.tokens = {}

    def add(self, sid, toks):
        self.tokens[sid] = list(toks)
        self.lib.add_sequence(sid, toks)
        self.orc.add_sequence(sid, toks)
        assert self.lib.can_allocate(sid) and self.orc.can_allocate(sid)
        self.lib.allocate(sid)
        self.orc.allocate(sid)
        return self.lib.sequence_info(sid)[1]          # cached tokens

    def remove(self, sid):
        self.lib.remove_sequence(sid)
        self.orc.remove_sequence(sid)

    def _qkv(self, sids, positions_per_seq):
        qs, ks, vs = [], [], []
        for sid, ps in zip(sids, positions_per_seq):
            for p in ps:
                q, k, v = token_qkv(self.tokens[sid][:p + 1])
                qs.append(q), ks.append(k), vs.append(v)
        return np.stack(qs), np.stack(ks), np.stack(vs)

    def _rotary(self, q, k, v, pos, slots):
        qr = pa.rotary_store_kvcache(dev_bf16(q), dev_bf16(k), dev_bf16(v), dev_i32(pos), self.dtable, self.dkc,
                                     self.dvc, dev_i32(slots))
        qr_o = self.oracle.rope_store_kvcache(q, k, v, pos, self.table, self.kc, self.vc, slots)
        return qr, qr_o

    def prefill(self, sids):
        m = self.lib.prepare_prefill(sids, MAXB)
        mo = self.orc.prepare_prefill(sids, MAXB)
        for key in mo:
            assert np.array_equal(m[key], mo[key]), key
        cq, ck = m["cu_seqlens_q"], m["cu_seqlens_k"]
        per_seq = [m["positions"][cq[r]:cq[r + 1]] for r in range(len(sids))]
        q, k, v = self._qkv(sids, per_seq)
        qr, qr_o = self._rotary(q, k, v, m["positions"], m["slot_mapping"])
        out = pa.prefill_varlen(qr, self.dkc, self.dvc, dev_i32(cq), dev_i32(ck), int(np.diff(cq).max()),
                                int(np.diff(ck).max()), dev_i32(m["block_tables"]), SCALE, True)
        _, ref = self.oracle.prefill_varlen(qr_o, self.kc, self.vc, cq, ck, m["block_tables"], SCALE, True,
                                            want_f64=True)
        torch.cuda.synchronize()
        assert_attention_close(out, ref, what=f"prefill {sids}")
        return m

    def decode(self, sids, next_tokens):
        for sid, t in zip(sids, next_tokens):
            self.tokens[sid].append(int(t))
            self.lib.append_token(sid, int(t))
            self.orc.append_token(sid, int(t))
            assert self.lib.can_append(sid) and self.orc.can_append(sid)
            self.lib.may_append(sid)
            self.orc.may_append(sid)
        m = self.lib.prepare_decode(sids, MAXB)
        mo = self.orc.prepare_decode(sids, MAXB)
        for key in mo:
            assert np.array_equal(m[key], mo[key]), key
        q, k, v = self._qkv(sids, [[p] for p in m["positions"]])
        qr, qr_o = self._rotary(q, k, v, m["positions"], m["slot_mapping"])
        L = int(m["context_lens"].max())
        out = pa.decode(qr, self.dkc, self.dvc, dev_i32(m["block_tables"]), dev_i32(m["context_lens"]), L, SCALE)
        _, ref = self.oracle.decode(qr_o, self.kc, self.vc, m["block_tables"], m["context_lens"], SCALE,
                                    want_f64=True)
        torch.cuda.synchronize()
        assert_attention_close(out, ref, what=f"decode {sids}")


def test_engine_flow_with_prefix_cache_growth_and_revival(oracle):
    rng = np.random.default_rng(2024)
    f = Flow(oracle)
    system = list(rng.integers(0, 500, 40))               # 2 full blocks + 8 tokens
    assert f.add(0, system + list(rng.integers(0, 500, 10))) == 0
    f.prefill([0])
    # two more requests behind the same system prompt: its 2 full blocks are cache hits
    assert f.add(1, system + list(rng.integers(0, 500, 23))) == 32
    assert f.add(2, system + list(rng.integers(0, 500, 5))) == 32
    m = f.prefill([1, 2])
    assert list(np.diff(m["cu_seqlens_q"])) == [31, 13]
    # decode across block boundaries (lengths 50, 63, 45 grow by 20)
    for _ in range(20):
        f.decode([0, 1, 2], rng.integers(0, 500, 3))
    # the first request finishes; a fourth one shares the still-used system blocks
    f.remove(0)
    assert f.add(3, system + [1, 2, 3]) == 32
    f.prefill([3])
    f.decode([1, 2, 3], rng.integers(0, 500, 3))
    # everything finishes; a new request revives the freed system blocks, whose K/V are still in the cache
    for s in (1, 2, 3):
        f.remove(s)
    assert f.lib.num_free_blocks() == NBLK
    assert f.add(4, system + list(rng.integers(0, 500, 30))) == 32
    f.prefill([4])
    for _ in range(5):
        f.decode([4], rng.integers(0, 500, 1))
    assert pa.device_error() == 0
