"""Packed segment table -> per-row (t, h, w) coordinates, exactly.

Definition followed:
* [P1] section 4: three-axis coordinates; video frames and audio samples share
  one physical timeline; left/right audio share t and differ on another axis;
  packed row order carries no position (the row permutation only moves rows).
* [P3] latent-frame passage: all 880 tokens of one latent frame carry the
  same t and differ only in (h, w).
* [P3] text passage: text tokens have t = index.  The workload descriptions
  place text at (i, i, i); the page's (i, 0, 0) is the "t-only" flag.
* [P3] chain ``position_ids[:, 0]`` is t: axis 0 = t, 1 = h, 2 = w.  The
  stereo channel goes on axis 2 (w) unless the channel-on-h flag is set.

Each coordinate is held as an exact rational num/den (int64); ``to_f32``
returns the correctly rounded (round-to-nearest-even) fp32 value of that
rational, computed with integer arithmetic only.

Normalised spatial canvas (video flag 4), from the [P3] passage on resolution:
the (h, w) grid is normalised by sqrt(H * W) and centred on [0, 32), so every
resolution covers the same range and a wide frame spans wider in w than in h
about the same midpoint.  Reading: cell centres y + 1/2 are measured from the
grid centre H/2, scaled by 32 / sqrt(H W), and moved to the midpoint 16:
    h = 16 + (y + 1/2 - H/2) * 32 / sqrt(H W),  w likewise with x and W.
The square root makes these irrational; ``packed_values`` evaluates them in
fp64 with the fixed operation order a = y + 0.5; b = a - 0.5 H;
s = 32 / sqrt(H W); h = 16 + b * s (each step one IEEE operation) and rounds
to fp32.
"""
from __future__ import annotations

import numpy as np

SEG_TEXT, SEG_VIDEO, SEG_AUDIO = 0, 1, 2
FLAG_TEXT_T_ONLY = 1
FLAG_AUDIO_CHANNEL_H = 2
FLAG_VIDEO_CANVAS = 4


def _field(seg, name, idx):
    return seg[idx] if isinstance(seg, (tuple, list)) else getattr(seg, name)


def _unpack(seg):
    names = ("kind", "count", "grid_h", "grid_w", "channels",
             "t_off_num", "t_step_num", "t_den", "flags")
    return tuple(int(_field(seg, n, i)) for i, n in enumerate(names))


def logical_coords(segments):
    """Exact coordinates of every logical element, in segment order.

    Returns (num, den): int64 arrays of shape [rows, 3] (axes t, h, w).
    """
    nums, dens = [], []
    for seg in segments:
        kind, count, gh, gw, ch, off, step, den, flags = _unpack(seg)
        if den <= 0 or count < 0:
            raise ValueError("bad segment")
        if kind == SEG_TEXT:
            i = np.arange(count, dtype=np.int64)
            t = off + i * step
            num = np.zeros((count, 3), np.int64)
            d = np.ones((count, 3), np.int64)
            num[:, 0], d[:, 0] = t, den
            if not flags & FLAG_TEXT_T_ONLY:          # (i, i, i)
                num[:, 1], d[:, 1] = t, den
                num[:, 2], d[:, 2] = t, den
        elif kind == SEG_VIDEO:
            if flags & FLAG_VIDEO_CANVAS:
                raise ValueError("canvas coordinates are irrational: use packed_values")
            k, y, x = np.meshgrid(np.arange(count), np.arange(gh), np.arange(gw), indexing="ij")
            k, y, x = (a.reshape(-1).astype(np.int64) for a in (k, y, x))
            num = np.stack([off + k * step, y, x], axis=1)
            d = np.ones_like(num)
            d[:, 0] = den
        elif kind == SEG_AUDIO:
            j, c = np.meshgrid(np.arange(count), np.arange(ch), indexing="ij")
            j, c = j.reshape(-1).astype(np.int64), c.reshape(-1).astype(np.int64)
            num = np.zeros((j.size, 3), np.int64)
            d = np.ones_like(num)
            num[:, 0], d[:, 0] = off + j * step, den
            if flags & FLAG_AUDIO_CHANNEL_H:
                num[:, 1] = c
            else:
                num[:, 2] = c
        else:
            raise ValueError(f"unknown segment kind {kind}")
        nums.append(num)
        dens.append(d)
    if not nums:
        return np.zeros((0, 3), np.int64), np.ones((0, 3), np.int64)
    return np.concatenate(nums), np.concatenate(dens)


def packed_coords(segments, perm=None):
    """Coordinates per PACKED row: row r takes logical element perm[r]."""
    num, den = logical_coords(segments)
    if perm is not None:
        perm = np.asarray(perm, np.int64)
        if sorted(perm.tolist()) != list(range(num.shape[0])):
            raise ValueError("perm is not a permutation of the logical rows")
        num, den = num[perm], den[perm]
    return num, den


def rational_to_f32(n: int, d: int) -> float:
    """Round the rational n/d to the nearest fp32, ties to even (normal range)."""
    n, d = int(n), int(d)
    if d == 0:
        raise ZeroDivisionError
    if n == 0:
        return 0.0
    neg = (n < 0) != (d < 0)
    n, d = abs(n), abs(d)
    # find e with 2^23 <= n / (d * 2^e) < 2^24
    e = n.bit_length() - d.bit_length() - 24
    while True:
        num = n << -e if e < 0 else n
        den = d << e if e > 0 else d
        if num < (den << 23):
            e -= 1
        elif num >= (den << 24):
            e += 1
        else:
            break
    q, r = divmod(num, den)
    if 2 * r > den or (2 * r == den and q & 1):
        q += 1
    v = float(q) * 2.0 ** e          # q <= 2^24: exact in fp64 and fp32
    return -v if neg else v


def to_f32(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    """Element-wise correctly rounded fp32 of num/den."""
    pairs = np.stack([num.reshape(-1), den.reshape(-1)], axis=1)
    uniq, inv = np.unique(pairs, axis=0, return_inverse=True)
    vals = np.array([rational_to_f32(a, b) for a, b in uniq], np.float32)
    return vals[inv.reshape(-1)].reshape(num.shape)


def to_f64(num: np.ndarray, den: np.ndarray) -> np.ndarray:
    """fp64 value of each exact rational (one correctly rounded division)."""
    return num.astype(np.float64) / den.astype(np.float64)


def canvas_f64(idx: np.ndarray, n: int, h: int, w: int) -> np.ndarray:
    """16 + (idx + 1/2 - n/2) * 32 / sqrt(h w) in fp64, one IEEE operation per step."""
    a = np.asarray(idx, np.float64) + 0.5
    b = a - 0.5 * float(n)
    s = 32.0 / np.sqrt(float(h) * float(w))
    return 16.0 + b * s


def logical_values(segments):
    """fp64 and fp32 coordinates of every logical element (any flags).

    Rational coordinates: fp64 = one correctly rounded division, fp32 =
    correctly rounded rational.  Canvas (h, w): fp64 by ``canvas_f64``,
    fp32 = round-to-nearest of that fp64 value.
    """
    f64s, f32s = [], []
    for seg in segments:
        kind, count, gh, gw, ch, off, step, den, flags = _unpack(seg)
        if kind == SEG_VIDEO and flags & FLAG_VIDEO_CANVAS:
            plain = (kind, count, gh, gw, ch, off, step, den, flags & ~FLAG_VIDEO_CANVAS)
            num, d = logical_coords([plain])
            v64 = to_f64(num, d)
            v32 = to_f32(num, d)
            y, x = num[:, 1], num[:, 2]
            v64[:, 1] = canvas_f64(y, gh, gh, gw)
            v64[:, 2] = canvas_f64(x, gw, gh, gw)
            v32[:, 1:] = v64[:, 1:].astype(np.float32)
        else:
            num, d = logical_coords([seg])
            v64, v32 = to_f64(num, d), to_f32(num, d)
        f64s.append(v64)
        f32s.append(v32)
    if not f64s:
        return np.zeros((0, 3)), np.zeros((0, 3), np.float32)
    return np.concatenate(f64s), np.concatenate(f32s)


def packed_values(segments, perm=None):
    """(fp64, fp32) coordinates per PACKED row (row r takes logical element perm[r])."""
    v64, v32 = logical_values(segments)
    if perm is not None:
        perm = np.asarray(perm, np.int64)
        if sorted(perm.tolist()) != list(range(v64.shape[0])):
            raise ValueError("perm is not a permutation of the logical rows")
        v64, v32 = v64[perm], v32[perm]
    return v64, v32
