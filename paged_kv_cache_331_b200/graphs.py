"""CUDA-graph capture of the decode step (store + decode, or rotary store + decode).

"Architektur im Überblick", section "CUDA Graph Optimierung": the engine
captures its decode step once per batch size in [1, 2, 4, 8] + [16, 32, ...,
max_bs], in descending order and into one shared memory pool, and replays
the smallest captured graph that holds the current batch.  This runner does
the same for the attention step of one layer: the new tokens' K/V rows are
scattered into the cache and every sequence attends over its blocks (one
launch, pa_store_decode).  Given
a rotary cos/sin cache, the step first rotates q and the new keys to their
positions ("Nano-vLLM 源碼學習", layers, 7 rotary_embedding.py), fused with the
store, and decode reads the rotated q.

Rows past the real batch are padding: their slot is -1 (the store skips them)
their context length 0 (decode writes zeros) and their position 0, so a padded replay computes
exactly what an unpadded call computes for the real rows.  The KV cache, the
static input buffers and the decode workspace keep their addresses for the
runner's lifetime: the captured kernels (and their TMA tensor maps) refer to
them.  Every step of the computation is a kernel of libpagedattn.so; torch
supplies the graph objects, buffers and streams.
"""
from __future__ import annotations

import bisect
import math

import torch

from . import _binding as pa


def graph_batch_sizes(max_bs: int):
    """[1, 2, 4, 8] + [16, 32, ..., max_bs] (sizes above max_bs dropped)."""
    return [b for b in [1, 2, 4, 8] + list(range(16, max_bs + 1, 16)) if b <= max_bs]


class DecodeGraphRunner:
    """Captured store_kvcache + decode steps for one layer's paged KV cache."""

    def __init__(self, k_cache, v_cache, num_heads, max_bs, max_blocks_per_seq, max_context_len, scale,
                 kv_chunk_size=0, cos_sin_cache=None):
        if not (k_cache.is_cuda and v_cache.is_cuda):
            raise TypeError("the KV cache must live on a CUDA device")
        self.k_cache, self.v_cache = k_cache, v_cache
        nb, bs_blk, hkv, d = k_cache.shape
        self.num_heads, self.num_kv_heads, self.head_dim, self.block_size = num_heads, hkv, d, bs_blk
        self.max_bs, self.max_blocks_per_seq = max_bs, max_blocks_per_seq
        self.max_context_len, self.scale, self.kv_chunk_size = max_context_len, scale, kv_chunk_size
        dev = k_cache.device
        bf = torch.bfloat16
        self.q = torch.zeros(max_bs, num_heads, d, dtype=bf, device=dev)
        self.new_k = torch.zeros(max_bs, hkv, d, dtype=bf, device=dev)
        self.new_v = torch.zeros(max_bs, hkv, d, dtype=bf, device=dev)
        self.slot_mapping = torch.full((max_bs,), -1, dtype=torch.int32, device=dev)
        self.block_tables = torch.full((max_bs, max_blocks_per_seq), -1, dtype=torch.int32, device=dev)
        self.context_lens = torch.zeros(max_bs, dtype=torch.int32, device=dev)
        self.out = torch.zeros(max_bs, num_heads, d, dtype=bf, device=dev)
        self.cos_sin_cache = cos_sin_cache
        self.positions = torch.zeros(max_bs, dtype=torch.int32, device=dev)
        self.q_rot = torch.zeros_like(self.q) if cos_sin_cache is not None else None
        self.graph_bs = graph_batch_sizes(max_bs)
        ws = max(pa.decode_workspace_size(b, num_heads, hkv, d, max_context_len, bs_blk, kv_chunk_size)
                 for b in self.graph_bs)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        self.graphs = {}
        self._capture()

    def _step(self, bs):
        if self.cos_sin_cache is None:     # one launch: the new rows are stored by the decode kernel itself
            pa.store_decode(self.q[:bs], self.new_k[:bs], self.new_v[:bs], self.slot_mapping[:bs], self.k_cache,
                            self.v_cache, self.block_tables[:bs], self.context_lens[:bs], self.max_context_len,
                            self.scale, out=self.out[:bs], workspace=self.workspace, kv_chunk_size=self.kv_chunk_size)
            return
        else:
            q = pa.rotary_store_kvcache(self.q[:bs], self.new_k[:bs], self.new_v[:bs], self.positions[:bs],
                                        self.cos_sin_cache, self.k_cache, self.v_cache, self.slot_mapping[:bs],
                                        out=self.q_rot[:bs])
        pa.decode(q, self.k_cache, self.v_cache, self.block_tables[:bs], self.context_lens[:bs],
                  self.max_context_len, self.scale, out=self.out[:bs], workspace=self.workspace,
                  kv_chunk_size=self.kv_chunk_size)

    def _capture(self):
        # one eager pass per size first: module loading and per-kernel set-up
        # (shared-memory attributes) happen outside any capture
        for bs in self.graph_bs:
            self._step(bs)
        torch.cuda.synchronize(self.k_cache.device)
        pool = None
        for bs in reversed(self.graph_bs):      # largest first, sharing one pool
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, pool=pool):
                self._step(bs)
            if pool is None:
                pool = g.pool()
            self.graphs[bs] = g

    def padded_size(self, n):
        i = bisect.bisect_left(self.graph_bs, n)
        if i == len(self.graph_bs):
            raise ValueError(f"batch of {n} exceeds the largest captured size {self.max_bs}")
        return self.graph_bs[i]

    def load(self, q, new_k, new_v, slot_mapping, block_tables, context_lens, positions=None):
        """Copy one step's inputs into the static buffers (padding the rest); returns the padded size.
        ``positions`` (the new tokens' positions) is required when the runner rotates."""
        n = q.shape[0]
        bs = self.padded_size(n)
        self.q[:n].copy_(q, non_blocking=True)
        self.new_k[:n].copy_(new_k, non_blocking=True)
        self.new_v[:n].copy_(new_v, non_blocking=True)
        self.slot_mapping[:n].copy_(slot_mapping, non_blocking=True)
        self.slot_mapping[n:bs].fill_(-1)
        w = block_tables.shape[1]
        if w > self.max_blocks_per_seq:
            raise ValueError("block tables are wider than the captured width")
        self.block_tables[:n, :w].copy_(block_tables, non_blocking=True)
        self.block_tables[:n, w:].fill_(-1)
        self.context_lens[:n].copy_(context_lens, non_blocking=True)
        self.context_lens[n:bs].fill_(0)
        if self.cos_sin_cache is not None:
            if positions is None:
                raise ValueError("a rotary runner needs the new tokens' positions")
            self.positions[:n].copy_(positions, non_blocking=True)
            self.positions[n:bs].fill_(0)
        return bs

    def replay(self, bs):
        self.graphs[bs].replay()

    def run(self, q, new_k, new_v, slot_mapping, block_tables, context_lens, positions=None):
        """Store the new rows and decode one step for a batch of q.shape[0] sequences; returns out[:n]."""
        bs = self.load(q, new_k, new_v, slot_mapping, block_tables, context_lens, positions)
        self.replay(bs)
        return self.out[:q.shape[0]]


class HostDecodeStep:
    """A decode step fed from and returned to host memory, as one CUDA graph.

    The step's inputs (q, the new K/V rows, their slots, the block tables and
    the context lengths) live in one pinned host buffer, so the graph is a single
    host-to-device copy, the fused store + decode (pa_store_decode), and a single
    device-to-host copy of the output.  The caller fills the host views returned
    by ``inputs()`` and calls ``run()``.  The KV cache stays on the device; its
    address is baked into the graph.
    """

    _ALIGN = 256

    def __init__(self, k_cache, v_cache, num_seqs, num_heads, max_blocks_per_seq, max_context_len, scale,
                 kv_chunk_size=0):
        nb, bs, hkv, d = k_cache.shape
        dev = k_cache.device
        B, hq = num_seqs, num_heads
        spec = [("q", (B, hq, d), torch.bfloat16), ("new_k", (B, hkv, d), torch.bfloat16),
                ("new_v", (B, hkv, d), torch.bfloat16), ("slot_mapping", (B,), torch.int32),
                ("block_tables", (B, max_blocks_per_seq), torch.int32), ("context_lens", (B,), torch.int32)]
        offs, o = [], 0
        for _, shape, dt in spec:
            n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
            offs.append((o, n))
            o = (o + n + self._ALIGN - 1) // self._ALIGN * self._ALIGN
        self.h2d_bytes = o
        self.host = torch.zeros(o, dtype=torch.uint8).pin_memory()
        self.dev = torch.zeros(o, dtype=torch.uint8, device=dev)

        def views(buf):
            return {name: buf[a:a + n].view(dt).view(shape) for (name, shape, dt), (a, n) in zip(spec, offs)}

        self._h, self._d = views(self.host), views(self.dev)
        self.out = torch.empty(B, hq, d, dtype=torch.bfloat16, device=dev)
        self.host_out = torch.empty(B, hq, d, dtype=torch.bfloat16).pin_memory()
        self.d2h_bytes = self.host_out.numel() * self.host_out.element_size()
        ws = pa.decode_workspace_size(B, hq, hkv, d, max_context_len, bs, kv_chunk_size)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)
        self.k_cache, self.v_cache = k_cache, v_cache
        self.max_context_len, self.scale, self.kv_chunk_size = max_context_len, scale, kv_chunk_size
        self._h["slot_mapping"].fill_(-1)            # an unfilled step stores nothing and reads nothing
        self._h["block_tables"].fill_(-1)
        self._step()                                   # eager once: kernel set-up happens outside the capture
        torch.cuda.synchronize(dev)
        self.graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(self.graph):
            self._step()

    def _step(self):
        d = self._d
        self.dev.copy_(self.host, non_blocking=True)
        pa.store_decode(d["q"], d["new_k"], d["new_v"], d["slot_mapping"], self.k_cache, self.v_cache,
                        d["block_tables"], d["context_lens"], self.max_context_len, self.scale, out=self.out,
                        workspace=self.workspace, kv_chunk_size=self.kv_chunk_size)
        self.host_out.copy_(self.out, non_blocking=True)

    def inputs(self):
        """Host views to fill before run(): q, new_k, new_v, slot_mapping, block_tables, context_lens."""
        return self._h

    def run(self):
        """Replay the step and wait for it; returns the host output [B, Hq, D] (bf16, pinned)."""
        self.graph.replay()
        torch.cuda.current_stream(self.out.device).synchronize()
        return self.host_out


class HostDecodePipeline:
    """Decode steps fed from and returned to host memory, with the copies of
    one step overlapping the kernels of its neighbours.

    A serving loop that gets each step's inputs from the host and hands each
    output back pays, per step, a host-to-device copy, the kernel and a
    device-to-host copy.  Run back to back on one stream they add up.  Here
    each of the ``depth`` slots has its own pinned and device buffers, and
    the three parts run on three streams:

        h2d stream:  copy inputs of step i (slot i % depth)
        compute:     pa_store_decode of step i (a CUDA graph per slot), after
                     that copy and after the output copy of step i - depth
        d2h stream:  copy the output of step i back, after its kernel

    so the input copy of step i+1 and the output copy of step i-1 run while
    the kernel of step i runs.  The kernels stay in order on one stream: each
    step stores its new rows before the next step reads the cache.

    Use: fill ``inputs(slot)`` for the slot ``next_slot()`` names, call
    ``submit()`` (returns a ticket), and ``wait(ticket)`` for the host output
    of that step.  Before a slot's inputs are filled again, the step that last
    used it must have been waited for (``submit`` checks this), since its copies
    read and write that slot's pinned buffers.
    """

    _ALIGN = 256

    def __init__(self, k_cache, v_cache, num_seqs, num_heads, max_blocks_per_seq, max_context_len, scale,
                 kv_chunk_size=0, depth=2):
        if depth < 1:
            raise ValueError("depth must be >= 1")
        nb, bs, hkv, d = k_cache.shape
        dev = k_cache.device
        B, hq = num_seqs, num_heads
        self.device, self.depth = dev, depth
        spec = [("q", (B, hq, d), torch.bfloat16), ("new_k", (B, hkv, d), torch.bfloat16),
                ("new_v", (B, hkv, d), torch.bfloat16), ("slot_mapping", (B,), torch.int32),
                ("block_tables", (B, max_blocks_per_seq), torch.int32), ("context_lens", (B,), torch.int32)]
        offs, o = [], 0
        for _, shape, dt in spec:
            n = math.prod(shape) * torch.empty((), dtype=dt).element_size()
            offs.append((o, n))
            o = (o + n + self._ALIGN - 1) // self._ALIGN * self._ALIGN
        self.h2d_bytes = o

        def views(buf):
            return {name: buf[a:a + n].view(dt).view(shape) for (name, shape, dt), (a, n) in zip(spec, offs)}

        self.host_in = [torch.zeros(o, dtype=torch.uint8).pin_memory() for _ in range(depth)]
        self.dev_in = [torch.zeros(o, dtype=torch.uint8, device=dev) for _ in range(depth)]
        self._h = [views(b) for b in self.host_in]
        self._d = [views(b) for b in self.dev_in]
        self.dev_out = [torch.empty(B, hq, d, dtype=torch.bfloat16, device=dev) for _ in range(depth)]
        self.host_out = [torch.empty(B, hq, d, dtype=torch.bfloat16).pin_memory() for _ in range(depth)]
        self.d2h_bytes = self.host_out[0].numel() * self.host_out[0].element_size()
        ws = pa.decode_workspace_size(B, hq, hkv, d, max_context_len, bs, kv_chunk_size)
        self.workspace = torch.empty(max(ws, 16), dtype=torch.uint8, device=dev)   # kernels are serialised
        self.k_cache, self.v_cache = k_cache, v_cache
        self.max_context_len, self.scale, self.kv_chunk_size = max_context_len, scale, kv_chunk_size
        for h in self._h:
            h["slot_mapping"].fill_(-1)            # an unfilled step stores nothing and reads nothing
            h["block_tables"].fill_(-1)
        for s in range(depth):
            self.dev_in[s].copy_(self.host_in[s])
        self.s_h2d = torch.cuda.Stream(dev)
        self.s_comp = torch.cuda.Stream(dev)
        self.s_d2h = torch.cuda.Stream(dev)
        ev = lambda: [torch.cuda.Event() for _ in range(depth)]   # noqa: E731
        self.h2d_done, self.comp_done, self.d2h_done = ev(), ev(), ev()
        self._submitted = 0
        self._waited = [True] * depth
        for s in range(depth):                      # eager once: kernel set-up happens outside the capture
            self._kernel(s)
        torch.cuda.synchronize(dev)
        self.graphs = []
        for s in range(depth):
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g):
                self._kernel(s)
            self.graphs.append(g)

    def _kernel(self, s):
        d = self._d[s]
        pa.store_decode(d["q"], d["new_k"], d["new_v"], d["slot_mapping"], self.k_cache, self.v_cache,
                        d["block_tables"], d["context_lens"], self.max_context_len, self.scale, out=self.dev_out[s],
                        workspace=self.workspace, kv_chunk_size=self.kv_chunk_size)

    def next_slot(self):
        return self._submitted % self.depth

    def inputs(self, slot):
        """Host views of a slot: q, new_k, new_v, slot_mapping, block_tables, context_lens."""
        return self._h[slot]

    def submit(self):
        """Enqueue the next step on the slot ``next_slot()`` names; returns its ticket."""
        s = self.next_slot()
        if not self._waited[s]:
            raise RuntimeError("the previous step on this slot has not been waited for")
        self._waited[s] = False
        cur = torch.cuda.current_stream(self.device)
        self.s_h2d.wait_stream(cur)                 # inputs the caller enqueued on its stream
        self.s_h2d.wait_event(self.comp_done[s])    # the kernel that last read this slot's device inputs
        with torch.cuda.stream(self.s_h2d):
            self.dev_in[s].copy_(self.host_in[s], non_blocking=True)
            self.h2d_done[s].record(self.s_h2d)
        self.s_comp.wait_event(self.h2d_done[s])
        self.s_comp.wait_event(self.d2h_done[s])    # the copy that last read this slot's device output
        with torch.cuda.stream(self.s_comp):
            self.graphs[s].replay()
            self.comp_done[s].record(self.s_comp)
        self.s_d2h.wait_event(self.comp_done[s])
        with torch.cuda.stream(self.s_d2h):
            self.host_out[s].copy_(self.dev_out[s], non_blocking=True)
            self.d2h_done[s].record(self.s_d2h)
        self._submitted += 1
        return self._submitted - 1

    def wait(self, ticket):
        """Block until step ``ticket`` is back in host memory; returns its output [B, Hq, D] (bf16, pinned),
        valid until the slot is submitted again."""
        s = ticket % self.depth
        self.d2h_done[s].synchronize()
        self._waited[s] = True
        return self.host_out[s]

    def join(self, stream=None):
        """Make ``stream`` (default: the current stream) wait for every submitted step."""
        stream = stream or torch.cuda.current_stream(self.device)
        for s in range(self.depth):
            stream.wait_event(self.d2h_done[s])
