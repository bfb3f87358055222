"""The whole packed MM-RoPE attention path, oracle side.

coords (exact rationals, evaluated in fp64) -> fp64 rotation of Q and K ->
fp64 exact softmax attention.  Inputs are the bf16 values themselves (the
oracle runs on the bf16-rounded inputs); the rotated Q/K stay in fp64 and are
never rounded.  Optional ``rows`` restricts the QUERY rows (all keys are
always used), which keeps full-size spot checks affordable.
"""
from __future__ import annotations

import numpy as np

from . import attention as _attn
from . import coords as _coords
from . import rope as _rope


def _as_f64(x: np.ndarray) -> np.ndarray:
    """bf16 bit patterns (uint16) or floating arrays -> fp64."""
    x = np.asarray(x)
    if x.dtype == np.uint16:
        return (x.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)
    return x.astype(np.float64)


def packed_angles(segments, perm, theta, sections, freq_rule=0):
    v64, _ = _coords.packed_values(segments, perm)
    return _rope.angles(v64, theta, sections, freq_rule)


def rotated_qk(segments, perm, q, k, theta=10000.0, sections=(32, 48, 48), pair_layout=0, freq_rule=0):
    """fp64 rotated (Q, K), each [N, H, D]."""
    ang = packed_angles(segments, perm, theta, sections, freq_rule)
    return (_rope.rotate(_as_f64(q), ang, pair_layout),
            _rope.rotate(_as_f64(k), ang, pair_layout))


def packed_mmrope_attention(segments, perm, q, k, v, theta=10000.0, sections=(32, 48, 48),
                            rows=None, heads=None, pair_layout=0, scale=None, freq_rule=0):
    """O [len(rows), len(heads), D] and LSE [len(heads), len(rows)] in fp64."""
    q = np.asarray(q)
    N, H, _ = q.shape
    rows = np.arange(N) if rows is None else np.asarray(rows, np.int64)
    heads = range(H) if heads is None else list(heads)
    ang = packed_angles(segments, perm, theta, sections, freq_rule)
    o = np.empty((rows.size, len(heads), v.shape[2]), np.float64)
    lse = np.empty((len(heads), rows.size), np.float64)
    for i, h in enumerate(heads):
        kr = _rope.rotate(_as_f64(k[:, h, :]), ang, pair_layout)
        qr = _rope.rotate(_as_f64(q[rows, h, :]), ang[rows], pair_layout)
        o[:, i], lse[i] = _attn.attention_head(qr, kr, _as_f64(v[:, h, :]), scale)
    return o, lse
