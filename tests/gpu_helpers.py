"""Shared helpers for the GPU parity tests: moving workloads to the device and
comparing with the oracle at the tolerance the path promises."""
import numpy as np
import torch

from paged_kv_cache_331_b200.workloads import bf16_bits_to_f32

# bf16 attention outputs against the float64 oracle
MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def dev_bf16(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)


def dev_i32(a: np.ndarray, device="cuda") -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a, dtype=np.int32)).to(device)


def host_bits(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16)


def host_f32(t: torch.Tensor) -> np.ndarray:
    return bf16_bits_to_f32(host_bits(t))


def assert_attention_close(gpu_out: torch.Tensor, ref_f64: np.ndarray, mask=None, what=""):
    got = host_f32(gpu_out).astype(np.float64)
    ref = np.asarray(ref_f64, dtype=np.float64)
    if mask is not None:
        got, ref = got[mask], ref[mask]
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max abs error {err.max():.3e} > {MAX_ABS}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean abs error {err.mean():.3e} > {MEAN_ABS}"
    return float(err.max()), float(err.mean())


class DeviceDecode:
    """A DecodeWorkload resident on the GPU."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.q = dev_bf16(w.q, device)
        self.k_cache = dev_bf16(w.k_cache, device)
        self.v_cache = dev_bf16(w.v_cache, device)
        self.new_k = dev_bf16(w.new_k, device)
        self.new_v = dev_bf16(w.new_v, device)
        self.slot_mapping = dev_i32(w.slot_mapping, device)
        self.block_tables = dev_i32(w.block_tables, device)
        self.context_lens = dev_i32(w.context_lens, device)


class DevicePrefill:
    """A PrefillWorkload resident on the GPU."""

    def __init__(self, w, device="cuda"):
        self.w = w
        self.q = dev_bf16(w.q, device)
        self.k_cache = dev_bf16(w.k_cache, device)
        self.v_cache = dev_bf16(w.v_cache, device)
        self.new_k = dev_bf16(w.new_k, device)
        self.new_v = dev_bf16(w.new_v, device)
        self.slot_mapping = dev_i32(w.slot_mapping, device)
        self.block_tables = dev_i32(w.block_tables, device)
        self.cu_seqlens_q = dev_i32(w.cu_seqlens_q, device)
        self.cu_seqlens_k = dev_i32(w.cu_seqlens_k, device)
