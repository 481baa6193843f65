"""Argument checks of the Python binding that run before anything reaches the
C ABI (CPU only): tensors on the wrong device or with the wrong shape are
rejected in Python, so a caller's mistake cannot become an out-of-bounds
access in a kernel."""
import pytest
import torch

from paged_kv_cache_331_b200 import _binding as B


def test_same_device():
    a, b = torch.empty(2), torch.empty(2)
    B._same_device(a, b=b, none=None)
    with pytest.raises(ValueError, match="meta"):
        B._same_device(a, m=torch.empty(2, device="meta"))


def test_shape_and_rows():
    t = torch.empty(4, 3, 8)
    B._shape(t, (4, 3, 8), "t")
    with pytest.raises(ValueError, match="shape"):
        B._shape(t, (4, 3, 16), "t")
    tables = torch.empty(5, 7, dtype=torch.int32)
    B._rows(tables, 5, "block_tables", 2)
    B._rows(tables, 3, "block_tables", 2)            # rows past the batch are not read
    with pytest.raises(ValueError, match="at least 6 rows"):
        B._rows(tables, 6, "block_tables", 2)
    with pytest.raises(ValueError, match="2-D"):
        B._rows(torch.empty(5, dtype=torch.int32), 5, "block_tables", 2)


def test_caches():
    kc = torch.empty(4, 16, 2, 64)
    B._caches(kc, torch.empty_like(kc), 64)
    with pytest.raises(ValueError, match="both"):
        B._caches(kc, torch.empty(3, 16, 2, 64))
    with pytest.raises(ValueError, match="both"):
        B._caches(torch.empty(4, 16, 128), torch.empty(4, 16, 128))
    with pytest.raises(ValueError, match="head_dim"):
        B._caches(kc, torch.empty_like(kc), 128)


def test_ops_reject_host_tensors():
    """Every op insists on CUDA tensors; on a host without a GPU that is where a call stops."""
    q = torch.empty(2, 4, 64, dtype=torch.bfloat16)
    kc = torch.empty(4, 16, 2, 64, dtype=torch.bfloat16)
    bt = torch.zeros(2, 4, dtype=torch.int32)
    cl = torch.ones(2, dtype=torch.int32)
    with pytest.raises(TypeError, match="CUDA"):
        B.decode(q, kc, kc, bt, cl, 16, 0.125)
    with pytest.raises(TypeError, match="CUDA"):
        B.store_kvcache(torch.empty(2, 2, 64, dtype=torch.bfloat16), torch.empty(2, 2, 64, dtype=torch.bfloat16),
                        kc, kc, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(TypeError, match="CUDA"):
        B.prefill_varlen(q, kc, kc, torch.zeros(2, dtype=torch.int32), torch.zeros(2, dtype=torch.int32), 1, 1, bt,
                         0.125)
    with pytest.raises(TypeError, match="CUDA"):
        B.merge_partials(torch.empty(2, 2, 4, 64), torch.empty(2, 2, 4))
