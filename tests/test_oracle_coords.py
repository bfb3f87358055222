"""Pins of the oracle's clock and coordinate decode (CPU only).

Each check ties the oracle to something the pages print or to an independent
enumeration, so that a wrong constant, axis or index fails here.
"""
from fractions import Fraction
import random

import numpy as np
import pytest

import workload as W
from oracle import clock, coords


# ------------------------------------------------------------------ clock --

def test_clock_matches_printed_values(golden):
    # one clock unit = one audio latent = 1/40 s; a 24 fps frame = 5/3 units
    assert clock.seconds(1) == Fraction(golden["clock_unit_seconds"])
    assert clock.ticks_per_source_frame() == Fraction(golden["ticks_per_source_frame"])
    assert clock.VIDEO_FPS == golden["source_fps"]
    assert clock.AUDIO_LATENT_HZ == golden["audio_latents_per_second"]
    assert clock.latent_frames_per_second() == golden["video_latents_per_second"]
    # the explainer's example: "video 3" is 0.5 s, "audio 3" is 0.075 s
    assert clock.seconds(3 * clock.ticks_per_latent_frame()) == Fraction(golden["video_latent_3_seconds"])
    assert clock.seconds(3) == Fraction(golden["audio_latent_3_seconds"])


def test_worked_example_counts(golden):
    h, w = golden["latent_sheet_hw"]
    assert tuple(golden["patch_thw"]) == clock.PATCH
    assert clock.tokens_per_latent_frame(h, w) == golden["tokens_per_latent_frame"]
    assert golden["latent_frames"] * clock.tokens_per_latent_frame(h, w) == golden["video_tokens"]
    assert clock.numbers_per_token() == golden["numbers_per_token"]
    assert clock.LATENT_CHANNELS == golden["latent_channels"]
    assert clock.VAE_SPATIAL * clock.PATCH[1] == golden["pixels_per_token_side"]
    assert clock.VAE_TEMPORAL_STRIDE == golden["vae_temporal"]
    assert clock.causal_latent_count(1) == golden["downsampler_single_frame_latents"]
    # 31 latents <-> 121 source frames (5.04 s at 24 fps); 91 <-> 361 (15.04 s)
    assert clock.causal_latent_count(121) == 31
    assert clock.causal_latent_count(361) == 91
    assert round(121 / 24, 2) == 5.04 and round(361 / 24, 2) == 15.04
    with pytest.raises(ValueError):
        clock.causal_latent_count(120)


def test_workload_tables_encode_the_pages_clock():
    step = clock.ticks_per_latent_frame()
    for wl in W.WORKLOADS:
        for s in wl.segments:
            if s.kind == W.SEG_VIDEO:
                assert Fraction(s.t_step_num, s.t_den) == step
            elif s.kind == W.SEG_AUDIO:
                assert Fraction(s.t_step_num, s.t_den) == 1 and s.channels == 2
            else:
                assert Fraction(s.t_step_num, s.t_den) == 1


def test_worked_example_segment_decodes_to_27280_rows(golden):
    wl = W.workload(2)
    vid = [s for s in wl.segments if s.kind == W.SEG_VIDEO]
    assert len(vid) == 1
    num, den = coords.logical_coords(vid)
    assert num.shape[0] == golden["video_tokens"]
    per = golden["tokens_per_latent_frame"]
    t = num[:, 0].reshape(golden["latent_frames"], per)
    assert (t == t[:, :1]).all(), "all tokens of one latent frame share t"
    assert len(np.unique(t[:, 0])) == golden["latent_frames"]
    hw = num[:per, 1:]
    assert len({tuple(x) for x in hw}) == per, "tokens of a frame differ in (h, w)"


def test_workload_row_totals():
    # totals stated in the five workload descriptions
    want = [82, 4584, 28196, 81792, 31952]
    for wl, n in zip(W.WORKLOADS, want):
        num, _ = coords.logical_coords(wl.segments)
        assert num.shape[0] == n == wl.n_rows


def _tiny_expected():
    """Independent enumeration of the tiny workload's logical coordinates."""
    out = []
    for i in range(16):                       # text at (i, i, i)
        out.append((Fraction(i), Fraction(i), Fraction(i)))
    for k in range(2):                        # 2 latent frames of a 4 x 6 grid
        for y in range(4):
            for x in range(6):
                out.append((Fraction(20 * k, 3), Fraction(y), Fraction(x)))
    for j in range(9):                        # 9 audio tokens x 2 channels
        for c in range(2):
            out.append((Fraction(j), Fraction(0), Fraction(c)))
    return out


def test_tiny_coords_brute_force():
    wl = W.workload(0)
    perm = W.permutation(wl)
    assert perm is not None and sorted(perm.tolist()) == list(range(82))
    num, den = coords.packed_coords(wl.segments, perm)
    exp = _tiny_expected()
    for r in range(82):
        got = tuple(Fraction(int(num[r, a]), int(den[r, a])) for a in range(3))
        assert got == exp[perm[r]], r


def test_audio_and_video_at_same_time_are_bit_identical():
    wl = W.workload(3)        # 91 latent frames and 600 audio tokens
    num, den = coords.logical_coords(wl.segments)
    f32 = coords.to_f32(num, den)
    first = {s: r for s, (r, _) in zip(range(len(wl.segments)), W.segment_row_ranges(wl))}
    vid0, aud0 = first[1], first[2]
    per = 22 * 40
    hits = 0
    for m in range(0, 31):
        k, j = 3 * m, 20 * m
        if k >= 91 or j >= 600:
            break
        tv = f32[vid0 + k * per, 0]
        ta = f32[aud0 + 2 * j, 0]
        assert tv.tobytes() == ta.tobytes()
        assert Fraction(int(num[vid0 + k * per, 0]), int(den[vid0 + k * per, 0])) == j
        hits += 1
    assert hits == 30


def test_stereo_channels_share_t_and_differ_on_w():
    seg = [W.audio(5, 2)]
    num, den = coords.logical_coords(seg)
    assert (num[0::2, 0] == num[1::2, 0]).all()
    assert (num[:, 1] == 0).all() and (num[0::2, 2] == 0).all() and (num[1::2, 2] == 1).all()
    num, _ = coords.logical_coords([W.audio(5, 2, flags=W.FLAG_AUDIO_CHANNEL_H)])
    assert (num[:, 2] == 0).all() and (num[1::2, 1] == 1).all()


def test_text_modes():
    num, den = coords.logical_coords([W.text(4)])
    assert num.tolist() == [[i, i, i] for i in range(4)]
    num, den = coords.logical_coords([W.text(4, flags=W.FLAG_TEXT_T_ONLY)])
    assert num.tolist() == [[i, 0, 0] for i in range(4)]


def test_negative_offsets_of_reference_segments():
    wl = W.workload(4)
    num, den = coords.logical_coords(wl.segments)
    ranges = W.segment_row_ranges(wl)
    # segment order: text, img0, aud0, img1, aud1, img2, aud2, img3..img8, video, audio
    img_t = []
    aud_t0 = []
    for s, (r0, n) in zip(wl.segments[1:], ranges[1:]):
        t = Fraction(int(num[r0, 0]), int(den[r0, 0]))
        if s.kind == W.SEG_VIDEO and s.count == 1:
            img_t.append(t)
        elif s.kind == W.SEG_AUDIO and s.count == 200:
            aud_t0.append(t)
    assert img_t == [-100 * (r + 1) for r in range(9)]
    assert aud_t0 == [-2000 * (c + 1) for c in range(3)]


# ------------------------------------------------------- fp32 rounding --

def _f32_neighbours(v):
    f = np.float32(v)
    return [np.nextafter(f, np.float32(-np.inf)), f, np.nextafter(f, np.float32(np.inf))]


def test_rational_to_f32_is_correctly_rounded():
    rng = random.Random(7)
    cases = [(20, 3), (-20, 3), (40, 3), (1, 3), (2 ** 24 + 1, 1), (2 ** 24 + 3, 1),
             (-6000, 1), (1820, 3), (-300, 3)]
    cases += [(rng.randint(-2 ** 24, 2 ** 24), rng.randint(1, 3 ** 9)) for _ in range(3000)]
    for n, d in cases:
        v = coords.rational_to_f32(n, d)
        q = Fraction(n, d)
        f = np.float32(v)
        assert float(f) == v
        errs = [abs(Fraction(float(x)) - q) for x in _f32_neighbours(v)]
        assert errs[1] <= errs[0] and errs[1] <= errs[2], (n, d)
        if errs[1] in (errs[0], errs[2]):             # a tie: the even one wins
            assert int(f.view(np.uint32)) % 2 == 0
    assert coords.rational_to_f32(2 ** 24 + 1, 1) == 2 ** 24       # tie -> even
    assert coords.rational_to_f32(2 ** 24 + 3, 1) == 2 ** 24 + 4   # tie -> even


def test_perm_must_be_a_permutation():
    with pytest.raises(ValueError):
        coords.packed_coords([W.text(3)], [0, 0, 1])
