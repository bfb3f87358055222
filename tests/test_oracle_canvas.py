"""Pins of the normalised spatial canvas mode (CPU only).

The explainer's passage on resolution states three properties, each checked
here on the oracle: the grid is centred on [0, 32) (midpoint 16; a square grid
stays inside (0, 32)); a 768p grid and a denser grid of the same aspect cover
the same range (only the sampling density changes); a wide frame spans wider
in w than in h about the same midpoint.
"""
import numpy as np
import pytest

import workload as W
from oracle import coords, pipeline


def _hw(grid_h, grid_w, frames=1):
    seg = W.video(frames, grid_h, grid_w, flags=W.FLAG_VIDEO_CANVAS)
    v64, v32 = coords.packed_values([seg])
    return v64, v32


@pytest.mark.parametrize("gh,gw", [(22, 40), (44, 80), (16, 16), (9, 16), (5, 3)])
def test_centred_on_16(gh, gw):
    v64, _ = _hw(gh, gw)
    assert abs(v64[:, 1].mean() - 16.0) < 1e-12 and abs(v64[:, 2].mean() - 16.0) < 1e-12


@pytest.mark.parametrize("n", [1, 2, 7, 22, 40, 160])
def test_square_grid_spans_inside_0_32(n):
    v64, _ = _hw(n, n)
    h = np.unique(v64[:, 1])
    assert h.min() > 0 and h.max() < 32
    np.testing.assert_allclose([h.min(), h.max()], [16.0 / n, 32.0 - 16.0 / n], atol=1e-12)
    np.testing.assert_allclose(np.diff(h), 32.0 / n, atol=1e-12)   # uniform spacing


def test_resolution_changes_density_not_range():
    lo, _ = _hw(22, 40)          # 704 x 1280 px at 32 px per token
    hi, _ = _hw(66, 120)         # same aspect, 3x denser (2K-like)
    for axis in (1, 2):
        a, b = np.unique(lo[:, axis]), np.unique(hi[:, axis])
        spacing = a[1] - a[0]
        assert b[1] - b[0] < spacing / 2                     # denser sampling
        assert abs((a.max() - a.min()) - (b.max() - b.min())) <= spacing   # same range
        assert abs(a.mean() - b.mean()) < 1e-12


def test_wide_frame_spans_wider_in_w():
    v64, _ = _hw(9, 16)
    h, w = np.unique(v64[:, 1]), np.unique(v64[:, 2])
    assert (w.max() - w.min()) > (h.max() - h.min())
    # one scale for both axes: equal spacing
    np.testing.assert_allclose(np.diff(h)[0], np.diff(w)[0], rtol=1e-14)


def test_t_axis_and_fp32_rounding():
    v64, v32 = _hw(4, 6, frames=3)
    num, den = coords.logical_coords([W.video(3, 4, 6)])
    np.testing.assert_array_equal(v32[:, 0], coords.to_f32(num, den)[:, 0])
    np.testing.assert_array_equal(v32[:, 1:], v64[:, 1:].astype(np.float32))


def test_rational_api_refuses_canvas():
    with pytest.raises(ValueError):
        coords.logical_coords([W.video(1, 2, 2, flags=W.FLAG_VIDEO_CANVAS)])


def test_pipeline_uses_canvas_values():
    segs = [W.text(4), W.video(2, 3, 5, flags=W.FLAG_VIDEO_CANVAS), W.audio(3, 2)]
    v64, _ = coords.packed_values(segs)
    ang = pipeline.packed_angles(segs, None, 10000.0, (32, 48, 48))
    np.testing.assert_array_equal(ang[:, 16], v64[:, 1])     # first h pair: inverse frequency 1
    np.testing.assert_array_equal(ang[:, 40], v64[:, 2])     # first w pair
