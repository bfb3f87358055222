"""Three-axis MM-RoPE in fp64.

Definition followed:
* [P1] section 4 and [P5] "H3-Omni-Transformer": Q and K are rotated by a
  three-axis (t, h, w) rotary position embedding.
* [P3] config passage: ``rope_theta`` and ``rope_freq_dim`` are configuration
  values and the inverse frequencies are computed from them, not stored.
  Reading used here: the head dimension is split into per-axis sections
  (t:32, h:48, w:48 dims) and axis a with D_a dims has the D_a/2 inverse
  frequencies theta^(-2j/D_a), j = 0 .. D_a/2 - 1 (freq_rule=0).
  The alternative reading (freq_rule=1): ``rope_freq_dim`` is the whole head
  dimension D, so pair p (counted over the head, t pairs first) has the one
  ladder's frequency theta^(-2p/D) and the sections only say which axis
  coordinate drives it.
* Rotary pair layout: adjacent dims (2p, 2p+1) form pair p; pairs 0..15 are
  t, 16..39 are h, 40..63 are w (pair_layout=0).  The alternative half-split
  layout pairs dim p with dim p + D/2 (pair_layout=1).
* Rotation of a pair (x0, x1) by angle a: (x0 cos a - x1 sin a,
  x0 sin a + x1 cos a), i.e. the complex product (x0 + i x1) e^{i a}.
"""
from __future__ import annotations

import numpy as np


def inv_freq(theta: float, sections=(32, 48, 48), freq_rule: int = 0):
    """Inverse frequencies of each axis's pairs, a list of three fp64 arrays.

    freq_rule 0: axis a restarts the ladder, theta^(-2j/D_a) for its D_a/2 pairs.
    freq_rule 1: one ladder theta^(-2p/D) over all D/2 pairs of the head, cut
    into the axes' consecutive slices.
    """
    for d_a in sections:
        if d_a % 2:
            raise ValueError("each axis needs an even number of dims")
    if freq_rule == 0:
        return [np.power(np.float64(theta), -2.0 * np.arange(d_a // 2, dtype=np.float64) / d_a)
                for d_a in sections]
    if freq_rule == 1:
        D = sum(sections)
        ladder = np.power(np.float64(theta), -2.0 * np.arange(D // 2, dtype=np.float64) / D)
        cut = np.cumsum([0] + [d_a // 2 for d_a in sections])
        return [ladder[cut[a]:cut[a + 1]] for a in range(len(sections))]
    raise ValueError("freq_rule must be 0 or 1")


def pair_table(theta: float, sections=(32, 48, 48), freq_rule: int = 0):
    """(axis[p], inv_freq[p]) for every rotary pair p = 0 .. D/2 - 1."""
    axes, freqs = [], []
    for a, f in enumerate(inv_freq(theta, sections, freq_rule)):
        axes.append(np.full(f.size, a, np.int64))
        freqs.append(f)
    return np.concatenate(axes), np.concatenate(freqs)


def angles(coords: np.ndarray, theta: float, sections=(32, 48, 48), freq_rule: int = 0) -> np.ndarray:
    """[rows, D/2] rotation angle of every pair: coords[r, axis[p]] * inv_freq[p]."""
    axis, freq = pair_table(theta, sections, freq_rule)
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
