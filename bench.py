#!/usr/bin/env python
"""Throughput of the paged-KV attention path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

A step is one decode step of the large-batch layer (256 sequences, context
U[100,1024] prompt + U[1,1024] generated, 32 q / 8 kv heads, head_dim 128,
block_size 256): store_kvcache of the 256 new K/V rows, then paged GQA decode
of every sequence, in one pa_store_decode launch.  It is the largest decode
workload that fits one GPU (~1.13 GB of KV per step, far more than L2), so
repeated steps read HBM; inputs are resident in HBM when the timed region
starts.  The headline value is decode KV bytes per second over all ranks.

The same JSON line carries, each with its own roofline:
  decode_workloads   the other decode workloads timed on their own: the tiny
                     4-sequence case (latency), the Qwen3-0.6B-shaped layer
                     (64 sequences) and the long-context split-KV case
                     (8 x 32768 + 1)
  store_256_rows     the headline step's 256-row store on its own (us, GB/s)
  prefill            the prefix-cached varlen prefill (32 sequences behind a
                     shared 1024-token prefix) in TFLOP/s, with its suffix store
  e2e                the headline step through host buffers (copies included)
  cpu_baseline       the oracle timed on the host cores

Under torchrun every rank runs its own independent batch (no collective on
the data path); the timed region is bracketed by barriers and the reported
time is the maximum over ranks.

--impl reference times the CPU oracle (float64, OpenMP) on the same workload
on rank 0 only.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import platform
import math
import os
import re
import subprocess
import sys
import threading
import time
from pathlib import Path

import numpy as np

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

METRIC = "decode KV bytes/s (% of HBM peak) and seqs/s; prefill TFLOP/s (% of peak)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}
PROFILES = ROOT / "profiles"
KERNEL_SOURCES = {
    "decode": ["paged_kv_cache_331_b200/csrc/decode.cu", "paged_kv_cache_331_b200/csrc/pa_device.cuh"],
    "prefill": ["paged_kv_cache_331_b200/csrc/prefill.cu", "paged_kv_cache_331_b200/csrc/pa_device.cuh"],
}


# ------------------------------------------------------------------------------------------ helpers --

def load_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        d["source"] = "measured"
        return d
    return dict(FALLBACK_PEAKS)


def kernel_source_hash(kind):
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kind]:
        h.update((ROOT / f).read_bytes())
    return h.hexdigest()[:16]


def profiled_traffic(kind, workload):
    """DRAM bytes per launch of the kernel on that workload, from an ncu capture summarised under profiles/, if the
    kernel's sources are unchanged since (same source hash); else None."""
    want = kernel_source_hash(kind)
    for f in sorted(PROFILES.glob("*.md")) + sorted(PROFILES.glob("*.txt")):
        for m in re.finditer(rf"traffic_per_launch\[{kind}:{re.escape(workload)}\]\s*=\s*([0-9.eE+]+)\s+"
                             rf"source_sha=([0-9a-f]+)", f.read_text()):
            if m.group(2) == want:
                return float(m.group(1))
    return None


def decode_algorithmic_bytes(w):
    """Bytes the decode step must move: every in-context K and V row once per kv head, q, out, tables."""
    L = w.context_lens.astype(np.int64)
    kv = int(L.sum()) * w.num_kv_heads * w.head_dim * 2 * 2
    qo = 2 * w.num_seqs * w.num_heads * w.head_dim * 2
    tables = int(np.ceil(L / w.block_size).sum()) * 4 + w.num_seqs * 4
    return kv, kv + qo + tables


def decode_store_bytes(w):
    """The new rows of a decode step: read and written once (K and V), plus their slots."""
    live = int((w.slot_mapping >= 0).sum())
    return live * w.num_kv_heads * w.head_dim * 2 * 2 * 2 + 4 * w.num_seqs


def prefill_flops(w):
    """4 * D * Hq per unmasked (query, key) pair: QK^T and PV, each a multiply-add."""
    total = 0
    for b in range(w.num_seqs):
        lq = int(w.cu_seqlens_q[b + 1] - w.cu_seqlens_q[b]); lk = int(w.cu_seqlens_k[b + 1] - w.cu_seqlens_k[b])
        if w.causal:
            total += lq * (lk - lq) + lq * (lq + 1) // 2
        else:
            total += lq * lk
    return 4 * w.head_dim * w.num_heads * total


class ClockSampler:
    """Samples SM clock, power and clock-event reasons while the timed region runs (NVML, nvidia-smi fallback)."""
    REASONS = {0x4: "sw_power_cap", 0x8: "hw_slowdown", 0x20: "sw_thermal_slowdown", 0x40: "hw_thermal_slowdown",
               0x80: "hw_power_brake_slowdown", 0x2: "applications_clocks_setting"}

    def __init__(self, torch_device_index, period_s=0.005):
        self.samples, self.max_mhz, self.err = [], None, None
        self.period = period_s
        self._stop = threading.Event()
        self._thread = None
        self._nvml = None
        try:
            import pynvml
            pynvml.nvmlInit()
            idx = torch_device_index
            vis = os.environ.get("CUDA_VISIBLE_DEVICES")
            if vis:
                ids = [v.strip() for v in vis.split(",") if v.strip()]
                if torch_device_index < len(ids) and ids[torch_device_index].isdigit():
                    idx = int(ids[torch_device_index])
            self._h = pynvml.nvmlDeviceGetHandleByIndex(idx)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self._h, pynvml.NVML_CLOCK_SM)
            self._nvml = pynvml
        except Exception as e:  # noqa: BLE001
            self.err = f"nvml: {e}"

    def _reasons(self):
        p = self._nvml
        fn = getattr(p, "nvmlDeviceGetCurrentClocksEventReasons", None) or p.nvmlDeviceGetCurrentClocksThrottleReasons
        return fn(self._h)

    def _run(self):
        p = self._nvml
        while not self._stop.is_set():
            try:
                self.samples.append((p.nvmlDeviceGetClockInfo(self._h, p.NVML_CLOCK_SM),
                                     p.nvmlDeviceGetPowerUsage(self._h) / 1000.0, int(self._reasons())))
            except Exception as e:  # noqa: BLE001
                self.err = str(e)
                return
            time.sleep(self.period)

    def __enter__(self):
        if self._nvml is not None:
            self._thread = threading.Thread(target=self._run, daemon=True)
            self._thread.start()
            t0 = time.perf_counter()       # running before the timed region starts: wait for its first samples
            while len(self.samples) < 2 and self.err is None and time.perf_counter() - t0 < 2.0:
                time.sleep(0.0005)
        return self

    def mark(self):
        """Index of the next sample (to tell which samples fall inside a timed region)."""
        return len(self.samples)

    def __exit__(self, *exc):
        self._stop.set()
        if self._thread:
            self._thread.join()

    def summary(self, lo=0, hi=None):
        samples = self.samples[lo:hi]
        if not samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0,
                    "note": self.err or "no samples"}
        mhz = [s[0] for s in samples]
        bits = 0
        for s in samples:
            bits |= s[2]
        reasons = sorted(name for bit, name in self.REASONS.items() if bits & bit)
        return {"sm_mhz": float(np.median(mhz)), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(samples), "power_w_max": round(max(s[1] for s in samples), 1)}


# ---------------------------------------------------------------------------------------- distributed --

def dist_setup(args):
    import torch
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl != "ours":
        return world, rank, local      # the reference arm runs on rank 0 alone and takes no collective step
    if world > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    else:
        torch.cuda.set_device(0)
    return world, rank, local


def barrier(world):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def _reduce(x, world, op):
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([float(x)], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=op)
    return float(t.item())


def max_over_ranks(x, world):
    """Slowest rank's value (timings are reported as the max over ranks)."""
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.MAX) if world > 1 else x


def sum_over_ranks(x, world):
    """Whole-job total (bytes and sequences processed by all ranks)."""
    import torch.distributed as dist
    return _reduce(x, world, dist.ReduceOp.SUM) if world > 1 else x


# -------------------------------------------------------------------------------------------- ours --

def to_dev(a, kind, dev):
    import torch
    if kind == "bf16":
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(dev)


def pinned(a, kind):
    import torch
    t = torch.from_numpy(np.ascontiguousarray(a).view(np.int16) if kind == "bf16"
                         else np.ascontiguousarray(a, dtype=np.int32))
    t = t.view(torch.bfloat16) if kind == "bf16" else t
    return t.pin_memory()


def decode_config(w, context_desc):
    """The workload as both arms name it: shapes, context distribution, pool and the KV bytes of one step."""
    kv, _ = decode_algorithmic_bytes(w)
    return {"workload": w.name, "num_seqs": w.num_seqs, "context_lens": context_desc, "num_heads": w.num_heads,
            "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim, "block_size": w.block_size,
            "pool_blocks": w.num_blocks, "kv_bytes_per_step": kv,
            "l2": (f"inputs larger than L2: {kv / 1e6:.0f} MB KV per step vs 126 MB L2" if kv > 126e6 else
                   f"{kv / 1e6:.2f} MB of KV: L2-resident between steps (a latency case)")}


HEADLINE = ("large_batch_decode", "U[100,1024] prompt + U[1,1024] generated")
DECODE_LEGS = {   # the other decode workloads, each timed as its own leg of the same run
    "tiny_decode": "{1,17,256,300}",
    "qwen3_decode": "U[128,4096]",
    "long_context_decode": "8 x 32768 + 1 x 1",
}


class DecodeOnDevice:
    """A decode workload resident on the GPU, with its output, workspace and chunk choice."""

    def __init__(self, w, dev, kv_chunk_size=0):
        import torch
        import paged_kv_cache_331_b200 as pa
        self.w = w
        self.q, self.kc, self.vc = to_dev(w.q, "bf16", dev), to_dev(w.k_cache, "bf16", dev), to_dev(w.v_cache, "bf16", dev)
        self.nk, self.nv = to_dev(w.new_k, "bf16", dev), to_dev(w.new_v, "bf16", dev)
        self.slots, self.bt = to_dev(w.slot_mapping, "i32", dev), to_dev(w.block_tables, "i32", dev)
        self.cl = to_dev(w.context_lens, "i32", dev)
        self.out = torch.empty_like(self.q)
        self.maxL = w.max_context_len
        self.chunk_arg = kv_chunk_size
        self.ws_bytes = pa.decode_workspace_size(w.num_seqs, w.num_heads, w.num_kv_heads, w.head_dim, self.maxL,
                                                 w.block_size, kv_chunk_size)
        self.ws = torch.empty(max(self.ws_bytes, 16), dtype=torch.uint8, device=dev)
        self.chunk = (pa.decode_chunk_size(w.num_seqs, w.num_kv_heads, self.maxL, w.block_size)
                      if kv_chunk_size == 0 else kv_chunk_size)
        nchunks = -(-self.maxL // self.chunk) if self.maxL else 1
        # one launch per step, plus the separate merge kernel above 16384 split sequences x kv heads
        self.launches_per_step = 1 + int(nchunks > 1 and w.num_seqs * w.num_kv_heads > 16384)

    def step(self):
        """One decode step: the new rows stored and every sequence decoded, in one pa_store_decode launch."""
        import paged_kv_cache_331_b200 as pa
        pa.store_decode(self.q, self.nk, self.nv, self.slots, self.kc, self.vc, self.bt, self.cl, self.maxL,
                        self.w.scale, out=self.out, workspace=self.ws, kv_chunk_size=self.chunk_arg)

    def store(self):
        import paged_kv_cache_331_b200 as pa
        pa.store_kvcache(self.nk, self.nv, self.kc, self.vc, self.slots)

    def decode(self):
        import paged_kv_cache_331_b200 as pa
        pa.decode(self.q, self.kc, self.vc, self.bt, self.cl, self.maxL, self.w.scale, out=self.out,
                  workspace=self.ws, kv_chunk_size=self.chunk_arg)


def timed_launches(fn, reps, dev, before=None):
    """Per-call CUDA-event times (ms) of fn on the current stream; `before` runs untimed ahead of each call."""
    import torch
    ev = []
    hold_gpu()
    for _ in range(reps):
        if before is not None:
            before()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); fn(); b.record()
        ev.append((a, b))
    torch.cuda.synchronize(dev)
    return [x.elapsed_time(y) for x, y in ev]


def decode_roofline(d, ms, peaks, kernel):
    """HBM roofline of one fused store + decode launch: algorithmic bytes / CUDA-event time."""
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    _, alg = decode_algorithmic_bytes(d.w)
    alg += decode_store_bytes(d.w)
    achieved = alg / (ms / 1e3) / 1e9
    return {"bound": "hbm", "kernel": kernel, "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
            "frac": round(achieved / hbm, 4), "algorithmic_bytes": alg, "launch_ms": round(ms, 5),
            "peak_kind": f"HBM copy ({peaks.get('source')})"}


def bench_decode_leg(name, desc, dev, peaks, reps, warmup):
    """One decode workload on its own: store + decode launches timed one by one (inputs larger than L2 except
    for the tiny workload, which is a latency case)."""
    import paged_kv_cache_331_b200 as pa
    from paged_kv_cache_331_b200 import workloads as W
    import torch
    w = W.WORKLOADS[name]()
    d = DecodeOnDevice(w, dev)
    for _ in range(warmup):
        d.step()
    if name == "tiny_decode":
        # a latency case: 50 steps captured in one CUDA graph and replayed, so the device time per step is
        # measured without the host's launch overhead (which dwarfs a kernel this small)
        torch.cuda.synchronize(dev)
        g = torch.cuda.CUDAGraph()
        n_graph = 50
        with torch.cuda.graph(g):
            for _ in range(n_graph):
                d.step()
        g.replay()
        ms_all = [t / n_graph for t in timed_launches(g.replay, max(3, reps // n_graph), dev)]
        eager = timed_launches(d.step, 20, dev)
    else:
        L2Flush(dev)()                 # the GPU stays busy while the host enqueues the first launches
        ms_all = timed_launches(d.step, reps, dev)
    assert pa.device_error() == 0
    ms = float(np.mean(ms_all))
    kv, _ = decode_algorithmic_bytes(w)
    res = {"config": decode_config(w, desc), "reps": reps, "ms": round(ms, 5), "ms_median": round(float(np.median(ms_all)), 5),
           "kv_gbs": round(kv / (ms / 1e3) / 1e9, 1), "seqs_per_s": round(w.num_seqs / (ms / 1e3), 1),
           "kv_chunk_size": d.chunk, "launches_per_step": d.launches_per_step,
           "roofline": decode_roofline(d, ms, peaks, "pa_store_decode")}
    res["roofline"]["traffic"] = profiled_traffic("decode", w.name)
    if name == "tiny_decode":
        res["latency_us"] = round(ms * 1e3, 2)
        res["eager_call_us"] = round(float(np.median(eager)) * 1e3, 2)
        res["note"] = ("latency case (294 KB of KV, L2-resident): latency_us is the device time per step of 50 "
                       "steps replayed from one CUDA graph; eager_call_us is one call from Python, host launch "
                       "overhead included; parity is its bar")
    return res, d


def bench_store_rows(d, dev, reps, flush):
    """store_kvcache of the workload's new rows on its own, L2 flushed (written, then evicted by a read) before
    every rep: microseconds and GB/s (2 MB cannot fill HBM within a launch's lifetime)."""
    import paged_kv_cache_331_b200 as pa
    for _ in range(3):
        d.store()
    ms_all = timed_launches(d.store, reps, dev, before=flush)
    assert pa.device_error() == 0
    ms = float(np.median(ms_all))
    nbytes = decode_store_bytes(d.w)
    return {"rows": int(d.w.num_seqs), "us": round(ms * 1e3, 2), "bytes": nbytes,
            "gbs": round(nbytes / (ms / 1e3) / 1e9, 1), "l2": "flushed before every rep"}


def bench_decode(args, world, rank, dev, peaks):
    """The headline: decode steps of the large-batch layer (256 sequences), timed as K consecutive steps."""
    import torch
    import paged_kv_cache_331_b200 as pa
    from paged_kv_cache_331_b200 import workloads as W

    w = W.large_batch_decode(seed=3 + 1000 * rank)
    d = DecodeOnDevice(w, dev)
    for _ in range(args.warmup):
        d.step()
    torch.cuda.synchronize(dev)
    K = args.steps
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(K)]
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(dev.index, period_s=0.0002)
    flush = L2Flush(dev)
    barrier(world)
    torch.cuda.synchronize(dev)
    with clk:
        # the flush and a short spin keep the GPU busy while the host enqueues the first steps, so the timed
        # region holds no launch gap; neither is part of the region
        flush()
        hold_gpu()
        i0 = clk.mark()
        t0.record()
        for i in range(K):
            ev[i][0].record()
            d.step()
            ev[i][1].record()
        t1.record()
        torch.cuda.synchronize(dev)
        i1 = clk.mark()
        # the same step as two calls (store kernel, then split + merge), for reference; the clock record goes on
        # over these reps, which run the same HBM-bound kernels at the same clocks
        Ku = max(3, min(K, 200))
        evu = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(Ku)]
        hold_gpu()
        for i in range(Ku):
            evu[i][0].record()
            d.store()
            evu[i][1].record()
            d.decode()
            evu[i][2].record()
        torch.cuda.synchronize(dev)
        more = max(0, 40 - K)                       # keep the record going for at least ~8 ms of steps
        for _ in range(more):
            d.step()
        torch.cuda.synchronize(dev)
    barrier(world)
    elapsed_ms = t0.elapsed_time(t1)
    decode_ms = float(np.mean([e[0].elapsed_time(e[1]) for e in ev]))
    assert pa.device_error() == 0
    elapsed_ms = max_over_ranks(elapsed_ms, world)
    unfused = {"store_ms": round(float(np.mean([e[0].elapsed_time(e[1]) for e in evu])), 5),
               "decode_ms": round(float(np.mean([e[1].elapsed_time(e[2]) for e in evu])), 5), "steps": Ku}

    kv_bytes, _ = decode_algorithmic_bytes(w)
    total_kv = sum_over_ranks(float(kv_bytes), world) * K
    value = total_kv / (elapsed_ms / 1e3) / 1e9
    seqs = sum_over_ranks(float(w.num_seqs), world) * K / (elapsed_ms / 1e3)
    roof = decode_roofline(d, decode_ms, peaks, "pa_store_decode (decode_split_kernel: store + decode)")
    roof["traffic"] = profiled_traffic("decode", w.name)

    # end to end through host buffers: every step copies q, the new K/V rows and the metadata (one packed pinned
    # buffer) to the device, runs the fused store + decode, and copies out back; the host waits for each step's
    # output one step behind, so a step's copies overlap the neighbouring steps' kernels
    from paged_kv_cache_331_b200.graphs import HostDecodePipeline
    pipe = HostDecodePipeline(d.kc, d.vc, w.num_seqs, w.num_heads, w.block_tables.shape[1], d.maxL, w.scale,
                              depth=3)
    for s in range(pipe.depth):
        hin = pipe.inputs(s)
        for name, arr in (("q", w.q), ("new_k", w.new_k), ("new_v", w.new_v)):
            hin[name].view(torch.int16).copy_(torch.from_numpy(np.ascontiguousarray(arr).view(np.int16)))
        hin["slot_mapping"].copy_(torch.from_numpy(w.slot_mapping))
        hin["block_tables"].copy_(torch.from_numpy(w.block_tables))
        hin["context_lens"].copy_(torch.from_numpy(w.context_lens))

    def e2e_run(n):
        tickets = []
        for i in range(n):
            if i >= pipe.depth:
                pipe.wait(tickets[i - pipe.depth])
            tickets.append(pipe.submit())
        for t in tickets[max(0, n - pipe.depth):]:
            pipe.wait(t)

    e2e_run(max(3, min(args.warmup, 10)))
    # at least 100 steps, so that the pipeline's fill (the first input copy) and drain (the last output copy)
    # weigh little against the steady state; every step's copies are inside the timed region
    Ke = max(100, min(K, 500))
    barrier(world)
    torch.cuda.synchronize(dev)
    s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    flush()
    s0.record()
    e2e_run(Ke)
    pipe.join()
    s1.record()
    torch.cuda.synchronize(dev)
    e2e_ms = max_over_ranks(s0.elapsed_time(s1), world)
    e2e_value = sum_over_ranks(float(kv_bytes), world) * Ke / (e2e_ms / 1e3) / 1e9
    assert pa.device_error() == 0
    clocks = clk.summary()
    clocks["window"] = ("the K timed steps, then the unfused reps and further steps of the same workload "
                        "(the same HBM-bound kernel)")
    clocks["timed_region"] = clk.summary(i0, i1)

    return w, d, {
        "value": value, "ms_per_step": elapsed_ms / K, "seqs_per_s": seqs, "unfused": unfused,
        "decode_ms": decode_ms, "kv_bytes_per_step": kv_bytes, "roofline": roof,
        "chunk": d.chunk, "ws_bytes": d.ws_bytes, "launches": d.launches_per_step * K,
        "clocks": clocks, "e2e": {"value": e2e_value, "unit": "GB/s", "h2d_bytes_per_step": pipe.h2d_bytes,
                                  "d2h_bytes_per_step": pipe.d2h_bytes, "steps": Ke,
                                  "how": "pinned host buffers; per step one H2D copy of the packed inputs, the fused "
                                         "store + decode, one D2H copy of out; three buffer slots on three streams so a "
                                         "step's copies overlap the neighbouring steps' kernels; the host waits for "
                                         "every step's output"},
    }


def hold_gpu(us=500.0):
    """Enqueue a spin kernel of about `us` microseconds (clock cycles at up to 2 GHz).  Placed just before a timed
    region, it keeps the GPU busy while the host queues the region's first launches, so that the first timed
    event does not wait on the host's launch overhead."""
    import torch
    sleep = getattr(torch.cuda, "_sleep", None)   # a spin kernel of N clock cycles
    if sleep is not None:
        sleep(int(us * 2000))


class L2Flush:
    """Flush between timed reps: write a buffer larger than L2 (126 MB), then read another one, so that the
    write-back of the flush's dirty lines happens before the timed region rather than inside it."""

    def __init__(self, dev, nbytes=256 << 20):
        import torch
        self.w = torch.empty(nbytes, dtype=torch.uint8, device=dev)
        self.r = torch.ones(nbytes // 4, dtype=torch.float32, device=dev)

    def __call__(self):
        self.w.zero_()
        return self.r.sum()


def bench_prefill(args, dev, peaks):
    import torch
    import paged_kv_cache_331_b200 as pa
    from paged_kv_cache_331_b200 import workloads as W

    w = W.prefix_prefill()
    q, kc, vc = to_dev(w.q, "bf16", dev), to_dev(w.k_cache, "bf16", dev), to_dev(w.v_cache, "bf16", dev)
    nk, nv = to_dev(w.new_k, "bf16", dev), to_dev(w.new_v, "bf16", dev)
    slots, bt = to_dev(w.slot_mapping, "i32", dev), to_dev(w.block_tables, "i32", dev)
    cq, ck = to_dev(w.cu_seqlens_q, "i32", dev), to_dev(w.cu_seqlens_k, "i32", dev)
    out = torch.empty_like(q)
    flush = L2Flush(dev)

    def store():
        pa.store_kvcache(nk, nv, kc, vc, slots)

    def prefill():
        pa.prefill_varlen(q, kc, vc, cq, ck, w.max_seqlen_q, w.max_seqlen_k, bt, w.scale, True, out=out)

    for _ in range(max(3, min(args.warmup, 10))):
        store(); prefill()
    torch.cuda.synchronize(dev)
    reps = max(3, min(args.steps, 100))
    st, pf = [], []
    hold_gpu()
    for _ in range(reps):
        flush()
        a, b, c = (torch.cuda.Event(enable_timing=True) for _ in range(3))
        a.record(); store(); b.record(); prefill(); c.record()
        st.append((a, b)); pf.append((b, c))
    torch.cuda.synchronize(dev)
    store_ms = float(np.median([x.elapsed_time(y) for x, y in st]))
    prefill_ms = float(np.median([x.elapsed_time(y) for x, y in pf]))
    assert pa.device_error() == 0
    flops = prefill_flops(w)
    tflops = flops / (prefill_ms / 1e3) / 1e12
    # the SM clock under a sustained prefill load: back-to-back launches for about half a second (K/V of this
    # workload stay in L2, so this is a clock record, not the reported time)
    sustained = None
    if not args.no_prefill_clock:
        n_sus = int(min(5000, max(50, 0.5 / (prefill_ms / 1e3))))
        s0, s1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        with ClockSampler(dev.index) as clk:
            s0.record()
            for _ in range(n_sus):
                prefill()
            s1.record()
            torch.cuda.synchronize(dev)
        assert pa.device_error() == 0
        sus_ms = s0.elapsed_time(s1) / n_sus
        sustained = {"launches": n_sus, "ms": sus_ms, "tflops": flops / (sus_ms / 1e3) / 1e12,
                     "note": "back to back, L2 warm", "clocks": clk.summary()}
    store_bytes = 2 * 2 * int(w.cu_seqlens_q[-1]) * w.num_kv_heads * w.head_dim * 2 + 4 * int(w.cu_seqlens_q[-1])
    store_gbs = store_bytes / (store_ms / 1e3) / 1e9
    rot = bench_rotary_store(w, dev, q, nk, nv, kc, vc, slots, flush, reps)
    big = bench_store_large(dev, reps)
    peak_tf = peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])
    return {
        "workload": w.name, "num_seqs": w.num_seqs, "prefix_len": 1024, "suffix": "U[64,512]",
        "l2": "flushed before every rep: a 256 MB buffer written, then another 256 MB read",
        "total_q": int(w.cu_seqlens_q[-1]), "ms": prefill_ms, "flops": flops, "tflops": tflops,
        "roofline": {"bound": "tensor", "achieved": tflops, "peak": peak_tf, "unit": "TFLOP/s",
                     "frac": tflops / peak_tf, "traffic": profiled_traffic("prefill", w.name),
                     "peak_kind": f"bf16 burst ({peaks.get('source')})"},
        "sustained": sustained,
        "store": {"rows": int(w.cu_seqlens_q[-1]), "ms": store_ms, "gbs": store_gbs,
                  "frac": store_gbs / peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]), "bytes": store_bytes},
        "rotary_store": rot,
        "store_large": big,
        "gpu_launches_per_rep": 2,
    }


def bench_store_large(dev, reps):
    """store_kvcache of 65 536 new rows of the large-batch layer shape (8 kv heads, head_dim 128): 256 MB read and
    256 MB written, more than L2 holds, so consecutive reps stream from HBM."""
    import torch
    import paged_kv_cache_331_b200 as pa
    n, hkv, d, bs = 65536, 8, 128, 256
    rng = np.random.default_rng(9)
    key = torch.randn(n, hkv, d, dtype=torch.bfloat16, device=dev)
    value = torch.randn(n, hkv, d, dtype=torch.bfloat16, device=dev)
    nb = n // bs + 16
    kc = torch.empty(nb, bs, hkv, d, dtype=torch.bfloat16, device=dev)
    vc = torch.empty_like(kc)
    slots = torch.from_numpy(rng.permutation(nb * bs)[:n].astype(np.int32)).to(dev)
    for _ in range(3):
        pa.store_kvcache(key, value, kc, vc, slots)
    torch.cuda.synchronize(dev)
    ev = []
    for _ in range(reps):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); pa.store_kvcache(key, value, kc, vc, slots); b.record()
        ev.append((a, b))
    torch.cuda.synchronize(dev)
    assert pa.device_error() == 0
    ms = float(np.median([x.elapsed_time(y) for x, y in ev]))
    nbytes = 2 * 2 * n * hkv * d * 2 + 4 * n
    gbs = nbytes / (ms / 1e3) / 1e9
    return {"rows": n, "ms": ms, "bytes": nbytes, "gbs": gbs,
            "frac": gbs / load_peaks().get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
            "note": "inputs larger than L2; random unique slots"}


def bench_rotary_store(w, dev, q, nk, nv, kc, vc, slots, flush, reps):
    """The prefill's new tokens through the fused rotary + store kernel (q rotated into a new buffer, rotated keys
    and values into the cache), L2 flushed (written, then evicted by a read) between reps."""
    import torch
    import paged_kv_cache_331_b200 as pa
    n = int(w.cu_seqlens_q[-1])
    lq = np.diff(w.cu_seqlens_q)
    cached = np.diff(w.cu_seqlens_k) - lq
    pos_h = np.concatenate([c + np.arange(l) for c, l in zip(cached, lq)]).astype(np.int32)
    max_pos = 40960
    table = pa.rotary_cos_sin_cache(max_pos, w.head_dim, 1e6, device=dev)
    pos = to_dev(pos_h, "i32", dev)
    q_rot = torch.empty_like(q)
    for _ in range(3):
        pa.rotary_store_kvcache(q, nk, nv, pos, table, kc, vc, slots, out=q_rot)
    torch.cuda.synchronize(dev)
    ev = []
    for _ in range(reps):
        flush()
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(); pa.rotary_store_kvcache(q, nk, nv, pos, table, kc, vc, slots, out=q_rot); b.record()
        ev.append((a, b))
    torch.cuda.synchronize(dev)
    assert pa.device_error() == 0
    ms = float(np.median([x.elapsed_time(y) for x, y in ev]))
    qb = n * w.num_heads * w.head_dim * 2
    kvb = n * w.num_kv_heads * w.head_dim * 2
    live = int((w.slot_mapping >= 0).sum())
    lkvb = live * w.num_kv_heads * w.head_dim * 2
    alg = (qb + 2 * kvb + 8 * n + len(np.unique(pos_h)) * w.head_dim * 4) + (qb + 2 * lkvb)
    gbs = alg / (ms / 1e3) / 1e9
    return {"tokens": n, "ms": ms, "bytes": alg, "gbs": gbs, "frac": gbs / load_peaks().get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]),
            "bytes_rule": "read q, k, v rows, positions, slots and each distinct table row once; write rotated q "
                          "and the stored k/v rows"}


def bench_graph(args, dev):
    """Store + decode of one layer at small batches, eager against a replayed CUDA graph (the engine's decode
    graphs): each step ends with a host synchronisation, as a token-by-token loop does, so the time includes
    the host's launch latency that the graph removes."""
    import torch
    import paged_kv_cache_331_b200 as pa
    from paged_kv_cache_331_b200 import workloads as W
    from paged_kv_cache_331_b200.graphs import DecodeGraphRunner

    res = {}
    for bs in (1, 8, 32):
        rng = np.random.default_rng(60 + bs)
        w = W.decode_workload(np.full(bs, 1024, np.int32), 16, 8, 128, 256, rng=rng)
        q, kc, vc = to_dev(w.q, "bf16", dev), to_dev(w.k_cache, "bf16", dev), to_dev(w.v_cache, "bf16", dev)
        nk, nv = to_dev(w.new_k, "bf16", dev), to_dev(w.new_v, "bf16", dev)
        slots, bt, cl = (to_dev(w.slot_mapping, "i32", dev), to_dev(w.block_tables, "i32", dev),
                         to_dev(w.context_lens, "i32", dev))
        out = torch.empty_like(q)
        ws = torch.empty(max(16, pa.decode_workspace_size(bs, 16, 8, 128, 1024, 256, 0)), dtype=torch.uint8,
                         device=dev)
        runner = DecodeGraphRunner(kc, vc, 16, max_bs=bs, max_blocks_per_seq=bt.shape[1], max_context_len=1024,
                                   scale=w.scale)
        pbs = runner.load(q, nk, nv, slots, bt, cl)

        def eager():
            pa.store_kvcache(nk, nv, kc, vc, slots)
            pa.decode(q, kc, vc, bt, cl, 1024, w.scale, out=out, workspace=ws)

        def graph():
            runner.replay(pbs)

        times = {}
        for name, fn in (("eager", eager), ("graph", graph)):
            for _ in range(5):
                fn()
            torch.cuda.synchronize(dev)
            n = max(20, min(args.steps, 300))
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            for _ in range(n):
                fn()
                torch.cuda.current_stream(dev).synchronize()
            b.record()
            torch.cuda.synchronize(dev)
            times[name] = a.elapsed_time(b) / n * 1e3
        assert torch.equal(out.view(torch.int16), runner.out[:bs].view(torch.int16))
        res[str(bs)] = {"eager_us": round(times["eager"], 2), "graph_us": round(times["graph"], 2)}
    assert pa.device_error() == 0
    return {"step": "store_kvcache + decode, context 1024, 16 q / 8 kv heads, D 128, host sync per step",
            "per_batch": res}


def cpu_baseline(w, budget_s=12.0):
    """The oracle as it stands, on this host's cores: store + decode of the same workload, repeated for about
    budget_s seconds."""
    from oracle import oracle as O
    orc = O.get()
    kc, vc = w.k_cache.copy(), w.v_cache.copy()
    kv_bytes, _ = decode_algorithmic_bytes(w)
    reps, t_total = 0, 0.0
    while t_total < budget_s and reps < 1000:
        t = time.perf_counter()
        orc.store_kvcache(w.new_k, w.new_v, kc, vc, w.slot_mapping)
        orc.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale)
        t_total += time.perf_counter() - t
        reps += 1
    # the same oracle on one thread, one rep of the decode (about a second)
    t = time.perf_counter()
    orc.decode(w.q, kc, vc, w.block_tables, w.context_lens, w.scale, nthreads=1)
    t1 = time.perf_counter() - t
    return {"value": kv_bytes * reps / t_total / 1e9, "unit": "GB/s", "cores": orc.max_threads(), "kind": "oracle",
            "sample": f"full workload (store + decode of all {w.num_seqs} sequences), {reps} rep(s), "
                      f"{t_total:.1f} s", "seconds": t_total, "cpu_model": cpu_model(),
            "one_thread": {"value": kv_bytes / t1 / 1e9, "unit": "GB/s", "sample": "one decode of the full workload",
                           "seconds": t1}}


def cpu_model():
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def run_ours(args, world, rank, local):
    import torch
    peaks = load_peaks()
    dev = torch.device("cuda", local if world > 1 else 0)
    import paged_kv_cache_331_b200 as pa
    pa.lib()
    w, d, res = bench_decode(args, world, rank, dev, peaks)
    legs, store3 = None, None
    if rank == 0 and not args.no_legs:
        flush = L2Flush(dev)
        store3 = bench_store_rows(d, dev, max(10, min(args.steps, 100)), flush)
        del d, flush
        torch.cuda.empty_cache()
        legs = {}
        only = set(args.legs.split(",")) if args.legs else None
        for name, desc in DECODE_LEGS.items():
            if only is not None and name not in only:
                continue
            reps = max(50, min(args.steps, 500)) if name != "tiny_decode" else 200
            legs[name], dl = bench_decode_leg(name, desc, dev, peaks, reps, max(3, args.warmup))
            del dl
            torch.cuda.empty_cache()
    pre = bench_prefill(args, dev, peaks) if (rank == 0 and not args.no_prefill) else None
    gr = bench_graph(args, dev) if (rank == 0 and not args.no_graph) else None
    cpu = cpu_baseline(w) if (rank == 0 and world == 1 and not args.no_cpu_baseline) else None
    if rank != 0:
        return
    hbm = peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"])
    config = decode_config(w, HEADLINE[1])
    config["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
    line = {
        "metric": METRIC, "value": round(res["value"], 2), "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(res["ms_per_step"], 5), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "accumulate": "f32",
        "data": "synthetic: seeded N(0,1) bf16 Q/K/V, block tables drawn from a shuffled 1.25x pool",
        "config": config,
        "step": f"store of the {w.num_seqs} new rows + decode of every sequence: one pa_store_decode launch "
                f"(kv_chunk_size {res['chunk']})",
        "seqs_per_s": round(res["seqs_per_s"], 1),
        "hbm_frac": round(res["value"] / world / hbm, 4),
        "roofline": res["roofline"],
        "unfused_step": res["unfused"],
        "e2e": res["e2e"], "gpu_launches": res["launches"], "clocks": res["clocks"],
    }
    if store3 is not None:
        line["store_256_rows"] = store3
    if legs is not None:
        line["decode_workloads"] = legs
    if pre is not None:
        line["prefill"] = pre
    if gr is not None:
        line["graph"] = gr
    if cpu is not None:
        line["cpu_baseline"] = cpu
        line["speedup_vs_cpu_baseline"] = round(res["value"] / cpu["value"], 1)
    print(json.dumps(line), flush=True)


# --------------------------------------------------------------------------------------- reference --

def run_reference(args, world, rank):
    """The CPU oracle on the host cores, each step a bounded sample of the same workload."""
    if rank != 0:
        return
    from oracle import oracle as O
    from paged_kv_cache_331_b200 import workloads as W
    orc = O.get()
    w = W.large_batch_decode()
    # calibrate: sequences per step so that warmup + steps end within about --reference-seconds
    one = W.decode_workload(w.context_lens[:1], w.num_heads, w.num_kv_heads, w.head_dim, w.block_size,
                            rng=np.random.default_rng(0))
    t = time.perf_counter()
    orc.decode(one.q, one.k_cache, one.v_cache, one.block_tables, one.context_lens, one.scale)
    mean_len = float(w.context_lens.mean())
    t1 = max(time.perf_counter() - t, 1e-4) * max(1.0, mean_len / float(one.context_lens[0]))
    per_step_budget = args.reference_seconds / max(1, args.steps + args.warmup)
    nseq = int(max(1, min(w.num_seqs, per_step_budget / t1)))
    sub = slice(0, nseq)
    kc, vc = w.k_cache.copy(), w.v_cache.copy()

    def step():
        orc.store_kvcache(w.new_k[sub], w.new_v[sub], kc, vc, w.slot_mapping[sub])
        orc.decode(w.q[sub], kc, vc, w.block_tables[sub], w.context_lens[sub], w.scale)

    for _ in range(args.warmup):
        step()
    t = time.perf_counter()
    for _ in range(args.steps):
        step()
    el = time.perf_counter() - t
    kv = int(w.context_lens[sub].astype(np.int64).sum()) * w.num_kv_heads * w.head_dim * 4
    value = kv * args.steps / el / 1e9
    sample = f"first {nseq} of {w.num_seqs} sequences per step (store + decode)"
    config = decode_config(w, HEADLINE[1])
    config["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(el / args.steps * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic: seeded N(0,1) bf16 Q/K/V, block tables drawn from a shuffled 1.25x pool",
        "config": config,
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": orc.max_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


def main():
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-graph", action="store_true")
    ap.add_argument("--legs", default="",
                    help="comma-separated decode legs to run (default: all of " + ", ".join(DECODE_LEGS) + ")")
    ap.add_argument("--no-legs", action="store_true",
                    help="skip the per-workload decode legs (tiny, Qwen3-shaped, long context) and the row store")
    ap.add_argument("--reference-seconds", type=float, default=120.0,
                    help="--impl reference: about how long the oracle's warm-up and timed steps take together")
    ap.add_argument("--no-prefill-clock", action="store_true",
                    help="skip the sustained prefill loop that records the SM clock under prefill load")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    world, rank, local = dist_setup(args)
    try:
        if args.impl == "reference":
            run_reference(args, world, rank)
        else:
            run_ours(args, world, rank, local)
    finally:
        if world > 1 and args.impl == "ours":
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
