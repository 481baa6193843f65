"""Error bound of the prefill kernel's FMA-pipe 2^x (CPU).

The prefill softmax evaluates a share of its exponentials as
2^x = 2^n * p(f), n = round(x), f = x - n in [-1/2, 1/2], p a cubic whose
coefficients are in csrc/prefill.cu.  This test reads those coefficients and
replays the same float32 steps in numpy (round-to-nearest via the 1.5*2^23
magic constant, Horner with fused multiply-adds modelled in float64 then
rounded, exponent add on the bit pattern) against 2**x.
"""
import re
from pathlib import Path

import numpy as np

SRC = Path(__file__).resolve().parent.parent / "paged_kv_cache_331_b200" / "csrc" / "prefill.cu"


def coeffs():
    text = SRC.read_text()
    c = [float(re.search(rf"kExpC{i}\s*=\s*([0-9.eE+-]+)f", text).group(1)) for i in range(4)]
    magic = float(re.search(r"kRoundMagic\s*=\s*([0-9.eE+-]+)f", text).group(1))
    return [np.float32(v) for v in c], np.float32(magic)


def fma32(a, b, c):
    return (a.astype(np.float64) * b.astype(np.float64) + c.astype(np.float64)).astype(np.float32)


def emulated_exp2(x):
    (c0, c1, c2, c3), magic = coeffs()
    x = np.maximum(x.astype(np.float32), np.float32(-125.0))
    t = (x + magic).astype(np.float32)
    n = (t - magic).astype(np.float32)
    f = fma32(n, np.full_like(n, -1.0), x)
    p = fma32(f, np.full_like(f, c3), np.full_like(f, c2))
    q = fma32(p, f, np.full_like(f, c1))
    r = fma32(q, f, np.full_like(f, c0))
    bits = r.view(np.int32) + (t.view(np.int32) << 23)
    return bits.view(np.float32)


def test_cubic_relative_error_on_reduced_range():
    (c0, c1, c2, c3), _ = coeffs()
    f = np.linspace(-0.5, 0.5, 100001).astype(np.float32)
    p = ((c3 * f + c2) * f + c1) * f + c0
    rel = np.abs(p.astype(np.float64) / np.exp2(f.astype(np.float64)) - 1)
    assert rel.max() < 1e-4


def test_full_range_against_exact_power_of_two():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.uniform(-125, 8, 200000), np.arange(-125, 9), np.arange(-125, 8) + 0.5,
                        [0.0, -0.0, 7.999, -124.9]]).astype(np.float32)
    got = emulated_exp2(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    assert np.all(np.isfinite(got)) and np.all(got > 0)
    assert np.max(np.abs(got / want - 1)) < 1e-4


def test_masked_inputs_give_negligible_weights():
    got = emulated_exp2(np.array([-np.inf, -1e30, -200.0, -126.0], np.float32)).astype(np.float64)
    assert np.all(got >= 0) and np.all(got < 2.0 ** -124)
