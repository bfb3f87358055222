"""Three-axis MM-RoPE in fp64.

Definition followed:
* [P1] section 4 and [P5] "H3-Omni-Transformer": Q and K are rotated by a
  three-axis (t, h, w) rotary position embedding.
* [P3] config passage: ``rope_theta`` and ``rope_freq_dim`` are configuration
  values and the inverse frequencies are computed from them, not stored.
  Reading used here: the head dimension is split into per-axis sections
  (t:32, h:48, w:48 dims) and axis a with D_a dims has the D_a/2 inverse
  frequencies theta^(-2j/D_a), j = 0 .. D_a/2 - 1.
* Rotary pair layout: adjacent dims (2p, 2p+1) form pair p; pairs 0..15 are
  t, 16..39 are h, 40..63 are w (pair_layout=0).  The alternative half-split
  layout pairs dim p with dim p + D/2 (pair_layout=1).
* Rotation of a pair (x0, x1) by angle a: (x0 cos a - x1 sin a,
  x0 sin a + x1 cos a), i.e. the complex product (x0 + i x1) e^{i a}.
"""
from __future__ import annotations

import numpy as np


def inv_freq(theta: float, sections=(32, 48, 48)):
    """Per-axis inverse frequencies, a list of three fp64 arrays."""
    out = []
    for d_a in sections:
        if d_a % 2:
            raise ValueError("each axis needs an even number of dims")
        j = np.arange(d_a // 2, dtype=np.float64)
        out.append(np.power(np.float64(theta), -2.0 * j / d_a))
    return out


def pair_table(theta: float, sections=(32, 48, 48)):
    """(axis[p], inv_freq[p]) for every rotary pair p = 0 .. D/2 - 1."""
    axes, freqs = [], []
    for a, f in enumerate(inv_freq(theta, sections)):
        axes.append(np.full(f.size, a, np.int64))
        freqs.append(f)
    return np.concatenate(axes), np.concatenate(freqs)


def angles(coords: np.ndarray, theta: float, sections=(32, 48, 48)) -> np.ndarray:
    """[rows, D/2] rotation angle of every pair: coords[r, axis[p]] * inv_freq[p]."""
    axis, freq = pair_table(theta, sections)
    return np.asarray(coords, np.float64)[:, axis] * freq[None, :]


def rotate(x: np.ndarray, ang: np.ndarray, pair_layout: int = 0) -> np.ndarray:
    """Rotate x [rows, ..., D] by ang [rows, D/2] (broadcast over heads)."""
    x = np.asarray(x, np.float64)
    D = x.shape[-1]
    half = D // 2
    if ang.shape[-1] != half:
        raise ValueError("angle table does not match head_dim")
    shape = (ang.shape[0],) + (1,) * (x.ndim - 2) + (half,)
    c = np.cos(ang).reshape(shape)
    s = np.sin(ang).reshape(shape)
    if pair_layout == 0:
        x0, x1 = x[..., 0::2], x[..., 1::2]
    elif pair_layout == 1:
        x0, x1 = x[..., :half], x[..., half:]
    else:
        raise ValueError("pair_layout must be 0 or 1")
    y0 = x0 * c - x1 * s
    y1 = x0 * s + x1 * c
    out = np.empty_like(x)
    if pair_layout == 0:
        out[..., 0::2], out[..., 1::2] = y0, y1
    else:
        out[..., :half], out[..., half:] = y0, y1
    return out
