"""Pins of the oracle's attention (CPU only): brute force, invariants, special cases."""
import numpy as np
import pytest

import workload as W
from oracle import attention, coords, pipeline, rope

THETA = 10000.0
SECTIONS = (32, 48, 48)


def _naive_longdouble(q, k, v, scale):
    """Full N x N matrix, softmax WITHOUT max subtraction, in long double."""
    q, k, v = (np.asarray(a, np.longdouble) for a in (q, k, v))
    e = np.exp((q @ k.T) * np.longdouble(scale))
    l = e.sum(axis=1, keepdims=True)
    return (e @ v) / l, np.log(l[:, 0])


@pytest.mark.parametrize("n", [1, 5, 82, 128])
def test_brute_force_tiny(n):
    rng = np.random.default_rng(n)
    q, k, v = (rng.standard_normal((n, 128)) for _ in range(3))
    o, lse = attention.attention_head(q, k, v, chunk=16)
    o_ref, lse_ref = _naive_longdouble(q, k, v, 1 / np.sqrt(128))
    np.testing.assert_allclose(o, o_ref.astype(np.float64), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse, lse_ref.astype(np.float64), rtol=0, atol=1e-12)


def test_brute_force_peaky_logits():
    # large logits: the max-subtracted form must still match the exact value
    rng = np.random.default_rng(11)
    q, k, v = rng.standard_normal((64, 128)) * 4, rng.standard_normal((64, 128)), rng.standard_normal((64, 16))
    o, _ = attention.attention_head(q, k, v)
    o_ref, _ = _naive_longdouble(q, k, v, 1 / np.sqrt(128))
    np.testing.assert_allclose(o, o_ref.astype(np.float64), rtol=0, atol=1e-11)


def test_default_scale_is_inverse_sqrt_head_dim():
    rng = np.random.default_rng(12)
    q, k, v = (rng.standard_normal((9, 128)) for _ in range(3))
    o1, _ = attention.attention_head(q, k, v)
    o2, _ = attention.attention_head(q, k, v, scale=128 ** -0.5)
    o3, _ = attention.attention_head(q, k, v, scale=1.0 / 128)
    np.testing.assert_allclose(o1, o2, rtol=0, atol=1e-14)
    assert np.abs(o1 - o3).max() > 1e-3


def test_constant_values_give_that_value():
    rng = np.random.default_rng(13)
    q, k = rng.standard_normal((30, 128)), rng.standard_normal((30, 128))
    c = rng.standard_normal(128)
    o, _ = attention.attention_head(q, k, np.tile(c, (30, 1)))
    np.testing.assert_allclose(o, np.tile(c, (30, 1)), atol=1e-12)


def test_single_key_gives_its_value():
    rng = np.random.default_rng(14)
    q, k, v = rng.standard_normal((7, 128)), rng.standard_normal((1, 128)), rng.standard_normal((1, 128))
    o, lse = attention.attention_head(q, k, v)
    np.testing.assert_allclose(o, np.tile(v, (7, 1)), atol=1e-15)
    np.testing.assert_allclose(lse, (q @ k[0]) / np.sqrt(128), atol=1e-12)


def test_permuting_rows_permutes_outputs():
    rng = np.random.default_rng(15)
    q, k, v = (rng.standard_normal((100, 2, 128)) for _ in range(3))
    p = rng.permutation(100)
    o, _ = attention.attention(q, k, v)
    op, _ = attention.attention(q[p], k[p], v[p])
    np.testing.assert_allclose(op, o[p], atol=1e-12)


def test_packed_row_order_carries_no_position():
    """The shuffled tiny workload equals the unshuffled one, rows permuted."""
    wl = W.workload(0)
    perm = W.permutation(wl)
    q, k, v = W.qkv_bf16(wl)
    o_s, _ = pipeline.packed_mmrope_attention(wl.segments, perm, q, k, v)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    # put the same per-element Q/K/V in logical order and run unshuffled
    o_u, _ = pipeline.packed_mmrope_attention(wl.segments, None, q[inv], k[inv], v[inv])
    np.testing.assert_allclose(o_s, o_u[perm], atol=1e-12)


@pytest.mark.parametrize("axis", [0, 1, 2])
def test_shifting_an_axis_leaves_outputs_unchanged(axis):
    wl = W.workload(0)
    num, den = coords.packed_coords(wl.segments, W.permutation(wl))
    c = coords.to_f64(num, den)
    q, k, v = (W.bf16_to_f64(a) for a in W.qkv_bf16(wl))
    outs = []
    for shift in (0.0, 37.0 / 3.0):
        cs = c.copy()
        cs[:, axis] += shift
        ang = rope.angles(cs, THETA, SECTIONS)
        o, _ = attention.attention(rope.rotate(q, ang), rope.rotate(k, ang), v)
        outs.append(o)
    np.testing.assert_allclose(outs[1], outs[0], atol=1e-9)
    # and a shift that is NOT common to all rows does change the output
    cs = c.copy()
    cs[: c.shape[0] // 2, axis] += 5.0
    ang = rope.angles(cs, THETA, SECTIONS)
    o, _ = attention.attention(rope.rotate(q, ang), rope.rotate(k, ang), v)
    assert np.abs(o - outs[0]).max() > 1e-3


def test_sampled_rows_match_full_rows():
    wl = W.workload(0)
    perm = W.permutation(wl)
    q, k, v = W.qkv_bf16(wl)
    o, lse = pipeline.packed_mmrope_attention(wl.segments, perm, q, k, v)
    rows = np.array([0, 5, 81])
    o2, lse2 = pipeline.packed_mmrope_attention(wl.segments, perm, q, k, v, rows=rows)
    # BLAS may block a 3-row product differently from an 82-row one
    np.testing.assert_allclose(o2, o[rows], rtol=0, atol=1e-14)
    np.testing.assert_allclose(lse2, lse[:, rows], rtol=0, atol=1e-14)


def test_zero_coordinates_give_plain_attention():
    rng = np.random.default_rng(16)
    q, k, v = (rng.standard_normal((20, 1, 128)) for _ in range(3))
    ang = rope.angles(np.zeros((20, 3)), THETA, SECTIONS)
    o, _ = attention.attention(rope.rotate(q, ang), rope.rotate(k, ang), v)
    o_ref, _ = _naive_longdouble(q[:, 0], k[:, 0], v[:, 0], 1 / np.sqrt(128))
    np.testing.assert_allclose(o[:, 0], o_ref.astype(np.float64), atol=1e-12)
