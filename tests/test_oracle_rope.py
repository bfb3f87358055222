"""Pins of the oracle's MM-RoPE (CPU only).

The rotation is checked against independent formulations: the complex-number
form of textbook 1-D RoPE (the text passage says the 3-D scheme reduces to
it), explicit dense rotation matrices (RoPE's relative form), norms and the
identity at coordinate zero.
"""
import cmath
import math

import numpy as np

import workload as W
from oracle import coords, pipeline, rope

THETA = 10000.0
SECTIONS = (32, 48, 48)


def _rng(seed=0):
    return np.random.default_rng(seed)


def test_pair_table_sections():
    axis, freq = rope.pair_table(THETA, SECTIONS)
    assert axis.size == 64
    assert (axis[:16] == 0).all() and (axis[16:40] == 1).all() and (axis[40:] == 2).all()
    # every axis restarts at frequency 1 and decays geometrically over its own dims
    for a, (lo, hi, d_a) in enumerate([(0, 16, 32), (16, 40, 48), (40, 64, 48)]):
        f = freq[lo:hi]
        assert f[0] == 1.0
        np.testing.assert_allclose(f[1:] / f[:-1], THETA ** (-2.0 / d_a), rtol=1e-14)
        np.testing.assert_allclose(f[-1], THETA ** (-(d_a - 2) / d_a), rtol=1e-14)


def _complex_rope_1d(x, pos, dims, base_dim):
    """Textbook RoPE (RoFormer) on x[dims], pairs (2i, 2i+1), as complex products."""
    y = np.array(x, np.float64)
    for i in range(dims // 2):
        z = complex(x[2 * i], x[2 * i + 1]) * cmath.exp(1j * pos * THETA ** (-2.0 * i / base_dim))
        y[2 * i], y[2 * i + 1] = z.real, z.imag
    return y


def test_text_only_reduces_to_1d_rope():
    n = 40
    x = _rng(1).standard_normal((n, 3, 128))
    num, den = coords.logical_coords([W.text(n, flags=W.FLAG_TEXT_T_ONLY)])
    ang = rope.angles(coords.to_f64(num, den), THETA, SECTIONS)
    y = rope.rotate(x, ang)
    for i in range(n):
        for h in range(3):
            want = _complex_rope_1d(x[i, h], i, 32, 32)
            np.testing.assert_allclose(y[i, h, :32], want[:32], rtol=0, atol=1e-12)
            assert (y[i, h, 32:] == x[i, h, 32:]).all(), "h/w dims untouched at h = w = 0"


def test_spatial_axes_rotate_their_own_sections():
    x = _rng(2).standard_normal(128)
    for axis, lo in ((1, 32), (2, 80)):
        c = np.zeros((1, 3))
        c[0, axis] = 7.0
        y = rope.rotate(x[None, :], rope.angles(c, THETA, SECTIONS))[0]
        want = _complex_rope_1d(x[lo:lo + 48], 7.0, 48, 48)
        np.testing.assert_allclose(y[lo:lo + 48], want, atol=1e-12)
        mask = np.ones(128, bool)
        mask[lo:lo + 48] = False
        assert (y[mask] == x[mask]).all()


def test_half_split_layout():
    x = _rng(3).standard_normal(128)
    c = np.array([[5.0, 0.0, 0.0]])
    y = rope.rotate(x[None, :], rope.angles(c, THETA, SECTIONS), pair_layout=1)[0]
    for p in range(64):
        f = THETA ** (-2.0 * p / 32) if p < 16 else 0.0
        z = complex(x[p], x[p + 64]) * cmath.exp(1j * 5.0 * f)
        assert abs(y[p] - z.real) < 1e-12 and abs(y[p + 64] - z.imag) < 1e-12


def test_rotation_preserves_pair_norms():
    x = _rng(4).standard_normal((50, 4, 128))
    c = _rng(5).uniform(-6000, 6000, (50, 3))
    y = rope.rotate(x, rope.angles(c, THETA, SECTIONS))
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12, atol=1e-12)


def _dense_rotation(delta):
    """128 x 128 block-diagonal rotation for a coordinate difference (t, h, w)."""
    R = np.zeros((128, 128))
    p = 0
    for axis, d_a in enumerate(SECTIONS):
        for j in range(d_a // 2):
            a = delta[axis] * THETA ** (-2.0 * j / d_a)
            c, s = math.cos(a), math.sin(a)
            R[2 * p, 2 * p], R[2 * p, 2 * p + 1] = c, -s
            R[2 * p + 1, 2 * p], R[2 * p + 1, 2 * p + 1] = s, c
            p += 1
    return R


def test_relative_form():
    rng = _rng(6)
    for _ in range(20):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        pq, pk = rng.uniform(-50, 50, 3), rng.uniform(-50, 50, 3)
        qr = rope.rotate(q[None], rope.angles(pq[None], THETA, SECTIONS))[0]
        kr = rope.rotate(k[None], rope.angles(pk[None], THETA, SECTIONS))[0]
        want = q @ _dense_rotation(pk - pq) @ k
        assert abs(qr @ kr - want) < 1e-10


def test_zero_coordinates_are_identity():
    x = _rng(7).standard_normal((3, 2, 128))
    y = rope.rotate(x, rope.angles(np.zeros((3, 3)), THETA, SECTIONS))
    assert (y == x).all()


def test_same_time_gives_identical_t_rotation():
    # video latent 3m and audio token 20m: identical rotation of the t dims
    wl = W.workload(1)
    num, den = coords.logical_coords(wl.segments)
    ang = rope.angles(coords.to_f64(num, den), THETA, SECTIONS)
    v0 = 128
    a0 = 128 + 5 * 880
    for m in range(2):
        rv, ra = v0 + 3 * m * 880, a0 + 2 * 20 * m
        assert (ang[rv, :16] == ang[ra, :16]).all()


def test_pipeline_rotated_qk_uses_packed_coords():
    wl = W.workload(0)
    perm = W.permutation(wl)
    q, k, _ = W.qkv_bf16(wl)
    qr, kr = pipeline.rotated_qk(wl.segments, perm, q, k)
    num, den = coords.packed_coords(wl.segments, perm)
    ang = rope.angles(coords.to_f64(num, den), THETA, SECTIONS)
    np.testing.assert_array_equal(qr, rope.rotate(W.bf16_to_f64(q), ang))
    # the permuted row r carries logical element perm[r]'s coordinates
    numl, denl = coords.logical_coords(wl.segments)
    assert (num == numl[perm]).all()


# ---- the single-ladder frequency reading (freq_rule=1) ----------------------

def test_single_ladder_pair_table():
    axis0, _ = rope.pair_table(THETA, SECTIONS)
    axis, freq = rope.pair_table(THETA, SECTIONS, freq_rule=1)
    assert (axis == axis0).all(), "the sections still assign the axes"
    # one geometric ladder over the whole head, no restart at the section edges
    assert freq[0] == 1.0
    np.testing.assert_allclose(freq[1:] / freq[:-1], THETA ** (-2.0 / 128), rtol=1e-14)
    np.testing.assert_allclose(freq[16], THETA ** (-32.0 / 128), rtol=1e-14)   # first h pair
    np.testing.assert_allclose(freq[40], THETA ** (-80.0 / 128), rtol=1e-14)   # first w pair


def test_single_ladder_text_is_full_head_1d_rope():
    # text rows sit at (i, i, i): with one ladder every pair sees the same
    # coordinate, which is textbook 1-D RoPE over all 128 dims
    n = 24
    x = _rng(11).standard_normal((n, 2, 128))
    num, den = coords.logical_coords([W.text(n)])
    ang = rope.angles(coords.to_f64(num, den), THETA, SECTIONS, freq_rule=1)
    y0 = rope.rotate(x, ang, pair_layout=0)
    y1 = rope.rotate(x, ang, pair_layout=1)
    for i in range(n):
        for h in range(2):
            np.testing.assert_allclose(y0[i, h], _complex_rope_1d(x[i, h], i, 128, 128), atol=1e-12)
            for p in range(64):
                z = complex(x[i, h, p], x[i, h, p + 64]) * cmath.exp(1j * i * THETA ** (-2.0 * p / 128))
                assert abs(y1[i, h, p] - z.real) < 1e-12 and abs(y1[i, h, p + 64] - z.imag) < 1e-12


def test_single_ladder_relative_form():
    rng = _rng(12)
    for _ in range(10):
        q, k = rng.standard_normal(128), rng.standard_normal(128)
        pq, pk = rng.uniform(-50, 50, 3), rng.uniform(-50, 50, 3)
        qr = rope.rotate(q[None], rope.angles(pq[None], THETA, SECTIONS, 1))[0]
        kr = rope.rotate(k[None], rope.angles(pk[None], THETA, SECTIONS, 1))[0]
        d = pk - pq
        R = np.zeros((128, 128))
        for p in range(64):
            a = d[0 if p < 16 else 1 if p < 40 else 2] * THETA ** (-p / 64.0)
            R[2 * p:2 * p + 2, 2 * p:2 * p + 2] = [[math.cos(a), -math.sin(a)], [math.sin(a), math.cos(a)]]
        assert abs(qr @ kr - q @ R @ k) < 1e-10


def test_unknown_freq_rule_is_an_error():
    import pytest
    with pytest.raises(ValueError):
        rope.inv_freq(THETA, SECTIONS, freq_rule=2)
