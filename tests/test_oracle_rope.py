"""Pins of the oracle's rotary position embedding (CPU only).

"Nano-vLLM 源碼學習", layers, 7 (rotary_embedding.py): RotaryEmbedding adds the
position to q and k through sines and cosines of the position.  The oracle reads
that as RoFormer's rotation with element i paired with element i + D/2 and
frequencies theta_i = base^(-2i/D).  These tests check it against what the
mathematics fixes: closed-form values of a worked example, the group law of
rotations, the complex-multiplication form, the relative-position property that
defines the method, norm preservation, position 0, and that the fused store writes
exactly the rotated key and the unchanged value.
"""
import numpy as np
import pytest

from paged_kv_cache_331_b200 import workloads as W

# cos and sin of 0.1 k and k (k = 1, 2, 3), closed-form values to 16 digits
_COS = {1: 0.5403023058681398, 2: -0.4161468365471424, 3: -0.9899924966004454,
        0.1: 0.9950041652780258, 0.2: 0.9800665778412416, 0.3: 0.9553364891256060}
_SIN = {1: 0.8414709848078965, 2: 0.9092974268256817, 3: 0.1411200080598672,
        0.1: 0.09983341664682815, 0.2: 0.19866933079506122, 0.3: 0.2955202066613396}


def _bits(rng, shape):
    return W.randn_bf16(rng, shape)


def _f(bits):
    return (bits.astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def test_rope_table_worked_example(oracle):
    # head_dim 4, base 100: theta_0 = 1 and theta_1 = 100^(-1/2) = 0.1
    t = oracle.rope_table(4, 4, 100.0)
    assert t[0].tolist() == [1.0, 1.0, 0.0, 0.0]
    for p in (1, 2, 3):
        want = [_COS[p], _COS[round(0.1 * p, 1)], _SIN[p], _SIN[round(0.1 * p, 1)]]
        np.testing.assert_allclose(t[p].astype(np.float64), want, rtol=0, atol=1.2e-7)


@pytest.mark.parametrize("d,base", [(64, 1e4), (128, 1e6)])
def test_rope_table_group_law(oracle, d, base):
    """e^{j m theta} e^{j n theta} = e^{j (m+n) theta} for every frequency."""
    t = oracle.rope_table(4096, d, base).astype(np.float64)
    z = t[:, : d // 2] + 1j * t[:, d // 2:]
    rng = np.random.default_rng(7)
    m = rng.integers(0, 2048, 200)
    n = rng.integers(0, 2048, 200)
    err = np.abs(z[m] * z[n] - z[m + n]).max()
    assert err < 4e-7
    assert np.abs(np.abs(z) - 1).max() < 1.2e-7


@pytest.mark.parametrize("d,base", [(64, 1e4), (128, 1e6)])
def test_rope_table_frequencies_are_geometric(oracle, d, base):
    """At position 1 the angles are theta_0 = 1 > theta_1 > ...: a geometric sequence whose ratio r
    satisfies r^(D/2) = base (so theta_{D/2} would be 1/base)."""
    t = oracle.rope_table(2, d, base).astype(np.float64)
    ang = np.arctan2(t[1, d // 2:], t[1, : d // 2])
    assert abs(ang[0] - 1.0) < 1e-7
    ratios = ang[:-1] / ang[1:]
    np.testing.assert_allclose(ratios, ratios.mean(), rtol=2e-5)
    np.testing.assert_allclose(ratios.mean() ** (d // 2), base, rtol=1e-3)


def _rope(oracle, x, positions, table, want_f64=True):
    """Rotate rows x [N, H, D] through the fused entry point with a throwaway cache (no stores)."""
    n, h, d = x.shape
    kc = np.zeros((1, 16, 1, d), np.uint16)
    key = np.zeros((n, 1, d), np.uint16)
    return oracle.rope_store_kvcache(x, key, key, positions, table, kc, kc.copy(), np.full(n, -1, np.int32),
                                     want_f64=want_f64)


@pytest.mark.parametrize("d", [64, 128])
def test_rope_is_complex_rotation_of_the_halves(oracle, d):
    rng = np.random.default_rng(11)
    table = oracle.rope_table(512, d, 1e4)
    x = _bits(rng, (6, 3, d))
    pos = rng.integers(0, 512, 6).astype(np.int32)
    out, of = _rope(oracle, x, pos, table)
    xf = _f(x)
    z = xf[..., : d // 2] + 1j * xf[..., d // 2:]
    w = (table[pos, : d // 2].astype(np.float64) + 1j * table[pos, d // 2:].astype(np.float64))[:, None, :]
    y = z * w
    np.testing.assert_allclose(of[..., : d // 2], y.real, rtol=0, atol=1e-12)
    np.testing.assert_allclose(of[..., d // 2:], y.imag, rtol=0, atol=1e-12)
    assert np.array_equal(out, oracle.bf16_round(of))


def test_rope_relative_position(oracle):
    """<R_m q, R_n k> = <R_{m-n} q, k>: the score depends on the offset only."""
    d = 128
    rng = np.random.default_rng(12)
    table = oracle.rope_table(4096, d, 1e6)
    q = _bits(rng, (32, 1, d))
    k = _bits(rng, (32, 1, d))
    m = rng.integers(0, 4096, 32).astype(np.int32)
    n = (m * rng.random(32)).astype(np.int32)
    _, rq = _rope(oracle, q, m, table)
    _, rk = _rope(oracle, k, n, table)
    _, rq_rel = _rope(oracle, q, (m - n).astype(np.int32), table)
    lhs = (rq * rk).sum(-1)
    rhs = (rq_rel * _f(k)).sum(-1)
    np.testing.assert_allclose(lhs, rhs, rtol=0, atol=2e-4)
    np.testing.assert_allclose(np.linalg.norm(rq, axis=-1), np.linalg.norm(_f(q), axis=-1), rtol=3e-7)


def test_rope_position_zero_is_identity(oracle):
    rng = np.random.default_rng(13)
    d, hq, hkv, bs = 64, 4, 2, 16
    table = oracle.rope_table(64, d, 1e4)
    q, key, val = _bits(rng, (3, hq, d)), _bits(rng, (3, hkv, d)), _bits(rng, (3, hkv, d))
    kc = np.zeros((2, bs, hkv, d), np.uint16)
    vc = np.zeros_like(kc)
    slots = np.array([0, 5, 17], np.int32)
    out = oracle.rope_store_kvcache(q, key, val, np.zeros(3, np.int32), table, kc, vc, slots)
    assert np.array_equal(out, q)
    assert np.array_equal(kc.reshape(-1, hkv, d)[slots], key)


def test_rope_positions_select_their_table_row(oracle):
    """Each token uses row positions[t] of the table and nothing else."""
    rng = np.random.default_rng(14)
    d = 64
    table = oracle.rope_table(300, d, 1e4)
    x = _bits(rng, (5, 2, d))
    pos = np.array([0, 299, 17, 17, 128], np.int32)
    out = _rope(oracle, x, pos, table, want_f64=False)
    for t in range(5):
        alone = _rope(oracle, x[t:t + 1], np.zeros(1, np.int32), table[pos[t]:pos[t] + 1].copy(), want_f64=False)
        assert np.array_equal(out[t], alone[0])


def test_rope_store_writes_rotated_key_and_raw_value(oracle):
    rng = np.random.default_rng(15)
    d, hq, hkv, bs, nb = 128, 8, 2, 16, 6
    n = 9
    table = oracle.rope_table(1024, d, 1e6)
    fused = _bits(rng, (n, (hq + 2 * hkv) * d))           # a fused QKV row, strided views as in the engine
    q = fused[:, : hq * d].reshape(n, hq, d)
    key = fused[:, hq * d:(hq + hkv) * d].reshape(n, hkv, d)
    val = fused[:, (hq + hkv) * d:].reshape(n, hkv, d)
    pos = rng.integers(0, 1024, n).astype(np.int32)
    slots = rng.permutation(nb * bs)[:n].astype(np.int32)
    slots[[2, 6]] = -1
    kc0 = np.full((nb, bs, hkv, d), 0x7FC0, np.uint16)    # NaN sentinel everywhere
    vc0 = kc0.copy()
    kc, vc = kc0.copy(), kc0.copy()
    out = oracle.rope_store_kvcache(q, key, val, pos, table, kc, vc, slots)
    krot = _rope(oracle, np.ascontiguousarray(key), pos, table, want_f64=False)
    assert np.array_equal(out, _rope(oracle, np.ascontiguousarray(q), pos, table, want_f64=False))
    kflat, vflat = kc.reshape(-1, hkv, d), vc.reshape(-1, hkv, d)
    live = slots >= 0
    assert np.array_equal(kflat[slots[live]], krot[live])
    assert np.array_equal(vflat[slots[live]], val[live])
    untouched = np.ones(nb * bs, bool)
    untouched[slots[live]] = False
    assert np.array_equal(kflat[untouched], kc0.reshape(-1, hkv, d)[untouched])
    assert np.array_equal(vflat[untouched], vc0.reshape(-1, hkv, d)[untouched])


def test_rope_rejects_positions_outside_the_table(oracle):
    table = oracle.rope_table(8, 64, 1e4)
    x = np.zeros((1, 1, 64), np.uint16)
    with pytest.raises(ValueError):
        _rope(oracle, x, np.array([8], np.int32), table)
    with pytest.raises(ValueError):
        _rope(oracle, x, np.array([-1], np.int32), table)
