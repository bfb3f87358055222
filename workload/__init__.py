"""Seeded synthetic workloads for packed MM-RoPE attention.

This module only describes and generates INPUTS: the packed segment tables of
the five workloads, bf16 Q/K/V drawn from a counter-based generator, the row
shuffle and the sampled query rows used for spot checks.  It holds none of the
method's arithmetic (no coordinate decode, no rotation, no softmax): the CPU
oracle and the CUDA library each implement those on their own, and both read
their inputs from here.

Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
number generators", OOPSLA 2014), in its counter form -- output n of a stream
seeded with s is mix(s + (n + 1) * GAMMA).  Normals come from the Box-Muller
transform in fp64, rounded to bf16 with round-to-nearest-even.

Segment tables follow the wording of the five workload descriptions:
text rows at coordinates (i, i, i); video latent frame k at t = 20k/3 with
(h, w) the patch-grid index; audio token j at t = j with the stereo channel on
the third axis; reference images and reference audio at fixed negative time
offsets.  A time value is stored as an exact rational
t = (t_off_num + idx * t_step_num) / t_den.
"""
from __future__ import annotations

import dataclasses
import os
from concurrent.futures import ThreadPoolExecutor
from typing import List, Sequence

import numpy as np

# ---------------------------------------------------------------- segments --

SEG_TEXT = 0
SEG_VIDEO = 1
SEG_AUDIO = 2

# Segment flags (bit set).
FLAG_TEXT_T_ONLY = 1        # text at (i, 0, 0) instead of (i, i, i)
FLAG_AUDIO_CHANNEL_H = 2    # stereo channel on the h axis instead of w
FLAG_VIDEO_CANVAS = 4       # (h, w) on the sqrt(H*W)-normalised [0, 32) canvas


@dataclasses.dataclass(frozen=True)
class Segment:
    """One contiguous run of logical elements of one modality.

    Logical element order inside a segment: text -> token index; video ->
    (frame, y, x) row-major; audio -> (token, channel).  The time of element
    index ``idx`` (token, frame or audio token) is the exact rational
    ``(t_off_num + idx * t_step_num) / t_den``.
    """
    kind: int
    count: int               # text tokens / latent frames / audio tokens
    grid_h: int = 0          # video patch grid
    grid_w: int = 0
    channels: int = 0        # audio channels (2 = stereo)
    t_off_num: int = 0
    t_step_num: int = 1
    t_den: int = 1
    flags: int = 0

    @property
    def rows(self) -> int:
        if self.kind == SEG_TEXT:
            return self.count
        if self.kind == SEG_VIDEO:
            return self.count * self.grid_h * self.grid_w
        if self.kind == SEG_AUDIO:
            return self.count * self.channels
        raise ValueError(f"unknown segment kind {self.kind}")

    def as_tuple(self):
        return (self.kind, self.count, self.grid_h, self.grid_w, self.channels,
                self.t_off_num, self.t_step_num, self.t_den, self.flags)


def text(count: int, flags: int = 0) -> Segment:
    """Text rows at t = i (and h = w = i unless FLAG_TEXT_T_ONLY)."""
    return Segment(SEG_TEXT, count, t_off_num=0, t_step_num=1, t_den=1, flags=flags)


def video(frames: int, grid_h: int, grid_w: int, t_off_num: int = 0, flags: int = 0) -> Segment:
    """Latent video frames at t = (t_off_num + 20 k) / 3, (h, w) = grid index."""
    return Segment(SEG_VIDEO, frames, grid_h, grid_w, 0, t_off_num, 20, 3, flags)


def audio(tokens: int, channels: int = 2, t_off: int = 0, flags: int = 0) -> Segment:
    """Audio latent tokens at t = t_off + j, channel on the third axis."""
    return Segment(SEG_AUDIO, tokens, 0, 0, channels, t_off, 1, 1, flags)


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    index: int
    heads: int
    head_dim: int
    segments: tuple
    shuffle: bool
    theta: float = 10000.0
    sections: tuple = (32, 48, 48)   # rotary dims on t, h, w

    @property
    def seed(self) -> int:
        return 1000 + self.index

    @property
    def n_rows(self) -> int:
        return sum(s.rows for s in self.segments)

    @property
    def attention_flops(self) -> int:
        """4 * N^2 * D * H: the two N x N x D contractions of full attention."""
        return 4 * self.n_rows * self.n_rows * self.head_dim * self.heads


def _ref2va_segments() -> tuple:
    # text, img0, aud0, img1, aud1, img2, aud2, img3 .. img8, target video, target audio
    segs: List[Segment] = [text(512)]
    for r in range(9):
        segs.append(video(1, 22, 40, t_off_num=-300 * (r + 1)))   # t = -100 (r + 1)
        if r < 3:
            segs.append(audio(200, 2, t_off=-2000 * (r + 1)))
    segs.append(video(25, 22, 40))
    segs.append(audio(160, 2))
    return tuple(segs)


WORKLOADS = (
    Workload("tiny", 0, 1, 128, (text(16), video(2, 4, 6), audio(9, 2)), shuffle=True),
    Workload("small", 1, 8, 128, (text(128), video(5, 22, 40), audio(28, 2)), shuffle=False),
    Workload("worked_example_27k", 2, 42, 128, (text(512), video(31, 22, 40), audio(202, 2)), shuffle=False),
    Workload("max_length_15s", 3, 42, 128, (text(512), video(91, 22, 40), audio(600, 2)), shuffle=False),
    Workload("ref2va", 4, 42, 128, _ref2va_segments(), shuffle=False),
)


def workload(i: int) -> Workload:
    return WORKLOADS[i]


def worked_example_resized(frames: int) -> Workload:
    """The worked-example layout (512 text rows, 22 x 40 latent frames, stereo
    audio, 42 x 128 heads) with ``frames`` latent frames and ceil(20 * frames / 3)
    audio tokens -- smaller or larger variants for profiling."""
    tokens = -(-20 * frames // 3)
    return Workload(f"worked_example_{frames}f", 2, 42, 128,
                    (text(512), video(frames, 22, 40), audio(tokens, 2)), shuffle=False)


# --------------------------------------------------------------- SplitMix64 --

GAMMA = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)

STREAM_Q, STREAM_K, STREAM_V, STREAM_PERM, STREAM_SAMPLE = 0, 1, 2, 3, 4


def _mix(z: np.ndarray) -> np.ndarray:
    z = z.copy()
    z ^= z >> np.uint64(30)
    z *= _M1
    z ^= z >> np.uint64(27)
    z *= _M2
    z ^= z >> np.uint64(31)
    return z


def splitmix64(seed: int, start: int, count: int) -> np.ndarray:
    """Outputs start .. start+count-1 of the SplitMix64 stream seeded with ``seed``."""
    with np.errstate(over="ignore"):
        n = np.arange(start + 1, start + count + 1, dtype=np.uint64)
        return _mix(np.uint64(seed & 0xFFFFFFFFFFFFFFFF) + n * GAMMA)


def stream_key(seed: int, stream: int) -> int:
    return int(splitmix64(seed, stream, 1)[0])


def _normals_chunk(key: int, first_pair: int, pairs: int) -> np.ndarray:
    x = splitmix64(key, 2 * first_pair, 2 * pairs).reshape(pairs, 2)
    u1 = ((x[:, 0] >> np.uint64(11)).astype(np.float64) + 1.0) * 2.0 ** -53   # (0, 1]
    u2 = (x[:, 1] >> np.uint64(11)).astype(np.float64) * 2.0 ** -53           # [0, 1)
    r = np.sqrt(-2.0 * np.log(u1))
    a = 2.0 * np.pi * u2
    out = np.empty((pairs, 2), np.float64)
    out[:, 0] = r * np.cos(a)
    out[:, 1] = r * np.sin(a)
    return out.reshape(-1)


def bf16_bits_rne(x: np.ndarray) -> np.ndarray:
    """fp64 -> bf16 bit patterns, round-to-nearest-even on 8 significant bits.

    Valid for finite inputs in the normal bf16 range (all generated values).
    """
    m, e = np.frexp(x)                       # x = m * 2^e, 0.5 <= |m| < 1
    m8 = np.rint(m * 256.0)                  # numpy rint rounds half to even
    y = np.ldexp(m8, e - 8).astype(np.float32)   # exact: 8 significant bits
    return (y.view(np.uint32) >> np.uint32(16)).astype(np.uint16)


def bf16_to_f64(bits: np.ndarray) -> np.ndarray:
    return (bits.astype(np.uint32) << np.uint32(16)).view(np.float32).astype(np.float64)


def normal_bf16(seed: int, stream: int, shape: Sequence[int], scale: float = 1.0,
                threads: int | None = None) -> np.ndarray:
    """bf16 bit patterns of ``scale`` * N(0,1), element e from pair e // 2."""
    total = int(np.prod(shape))
    assert total % 2 == 0
    key = stream_key(seed, stream)
    out = np.empty(total, np.uint16)
    pairs = total // 2
    chunk = 1 << 21
    starts = list(range(0, pairs, chunk))

    def work(p0: int) -> None:
        n = min(chunk, pairs - p0)
        out[2 * p0: 2 * (p0 + n)] = bf16_bits_rne(scale * _normals_chunk(key, p0, n))

    threads = threads or min(16, os.cpu_count() or 1)
    if len(starts) == 1:
        work(0)
    else:
        with ThreadPoolExecutor(threads) as ex:
            list(ex.map(work, starts))
    return out.reshape(shape)


def qkv_bf16(w: Workload, q_scale: float = 1.0):
    """Q, K, V as uint16 bf16 bit arrays of shape [N, H, D] (packed row order)."""
    shape = (w.n_rows, w.heads, w.head_dim)
    q = normal_bf16(w.seed, STREAM_Q, shape, q_scale)
    k = normal_bf16(w.seed, STREAM_K, shape)
    v = normal_bf16(w.seed, STREAM_V, shape)
    return q, k, v


def uniform01(seed: int, stream: int, count: int) -> np.ndarray:
    x = splitmix64(stream_key(seed, stream), 0, count)
    return (x >> np.uint64(11)).astype(np.float64) * 2.0 ** -53


def permutation(w: Workload) -> np.ndarray | None:
    """Packed row r -> logical element perm[r]; None when rows are in segment order.

    Fisher-Yates (Knuth, TAOCP vol. 2, Algorithm 3.4.2P) driven by the stream.
    """
    if not w.shuffle:
        return None
    return fisher_yates(w.n_rows, w.seed, STREAM_PERM)


def fisher_yates(n: int, seed: int, stream: int = STREAM_PERM) -> np.ndarray:
    perm = np.arange(n, dtype=np.int32)
    u = uniform01(seed, stream, max(n, 1))
    for i in range(n - 1, 0, -1):
        j = int(u[n - 1 - i] * (i + 1))
        perm[i], perm[j] = perm[j], perm[i]
    return perm


def segment_row_ranges(w: Workload):
    """[(first_logical_row, rows)] per segment, in segment order."""
    out, r = [], 0
    for s in w.segments:
        out.append((r, s.rows))
        r += s.rows
    return out


def sample_rows(w: Workload, n: int, tile: int = 128) -> np.ndarray:
    """Seeded sorted sample of packed query rows for spot checks at full size.

    Always includes rows 0 and N-1, the whole last partial 128-row tile, the
    first and last row of every segment (mapped through the row permutation)
    and ``n`` seeded draws.
    """
    N = w.n_rows
    perm = permutation(w)
    inv = None
    if perm is not None:
        inv = np.empty(N, np.int64)
        inv[perm] = np.arange(N)
    pick = {0, N - 1}
    last_tile = (N - 1) // tile * tile
    pick.update(range(last_tile, N))
    for first, rows in segment_row_ranges(w):
        for lr in (first, first + rows - 1, first + rows // 2):
            pick.add(int(inv[lr]) if inv is not None else lr)
    u = uniform01(w.seed, STREAM_SAMPLE, n)
    pick.update(int(x) for x in (u * N).astype(np.int64))
    return np.array(sorted(pick), dtype=np.int64)
