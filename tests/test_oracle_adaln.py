"""Pins of the AdaLN oracle (CPU only): closed forms and the index rule."""
import numpy as np
import pytest

from oracle import adaln


def _rng(s=0):
    return np.random.default_rng(s)


def test_index_rule_from_the_page():
    # adaln_indices = timestep_indices * 3 + token_tags
    ts = np.array([0, 0, 0, 1, 1, 4])
    tags = np.array([0, 1, 2, 0, 2, 1])
    assert adaln.adaln_index(ts, tags).tolist() == [0, 1, 2, 3, 5, 13]


def test_zero_modulation_is_plain_layer_norm():
    x = _rng(1).standard_normal((7, 96)) * 3 + 5
    y = adaln.adaln_modulate(x, np.zeros(7, int), np.zeros(7, int), np.zeros((1, 2, 96)), eps=0.0)
    np.testing.assert_allclose(y.mean(axis=1), 0, atol=1e-12)
    np.testing.assert_allclose(y.var(axis=1), 1, atol=1e-12)


def test_scale_minus_one_gives_the_shift():
    x = _rng(2).standard_normal((4, 64))
    table = np.zeros((3, 2, 64))
    table[2, 0] = np.arange(64)
    table[2, 1] = -1.0
    y = adaln.adaln_modulate(x, np.zeros(4, int), np.full(4, 2), table)
    np.testing.assert_allclose(y, np.tile(np.arange(64.0), (4, 1)), atol=1e-12)


def test_each_row_gathers_its_own_entry():
    n, c = 30, 48
    rng = _rng(3)
    x = rng.standard_normal((n, c))
    ts, tags = rng.integers(0, 4, n), rng.integers(0, 3, n)
    table = rng.standard_normal((12, 2, c))
    y = adaln.adaln_modulate(x, ts, tags, table)
    for r in range(n):
        e = 3 * ts[r] + tags[r]
        xr = x[r]
        norm = (xr - xr.mean()) / np.sqrt(((xr - xr.mean()) ** 2).mean() + 1e-6)
        np.testing.assert_allclose(y[r], norm * (1 + table[e, 1]) + table[e, 0], atol=1e-12)


def test_shift_and_scale_invariance_of_the_norm():
    x = _rng(4).standard_normal((5, 80))
    a = adaln.layer_norm(x)
    b = adaln.layer_norm(3.0 * x + 7.0)
    np.testing.assert_allclose(a, b, atol=1e-5)        # eps breaks exact equality slightly


def test_out_of_range_entry_is_an_error():
    with pytest.raises(IndexError):
        adaln.adaln_modulate(np.zeros((1, 8)), [1], [0], np.zeros((3, 2, 8)))
