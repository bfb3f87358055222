"""The shared physical clock and token-count facts, as the pages state them.

[P1] section 4 and the [P3] clock-unit passage: one clock unit is one audio
latent, i.e. 1/40 s; a 24 fps source frame lasts (1/24) / (1/40) = 5/3 units.
[P3] passage on video vs audio rates: video yields 6 latent frames per second
(4x temporal compression of 24 fps), audio 40 latents per second.
[P3] causal-downsampler passage: T source frames -> (T - 1)/r + 1 latents.
[P3] patchify passage: a 1x2x2 patch of 24-channel cells is 96 numbers.
[P3] latent-frame passage: a 44 x 80 latent sheet patchified 1x2x2 is
22 x 40 = 880 tokens, all with the same time coordinate.
"""
from fractions import Fraction

AUDIO_LATENT_HZ = 40          # clock ticks per second
VIDEO_FPS = 24                # source frames per second
VAE_TEMPORAL_STRIDE = 4       # source frames per latent frame (after the first)
VAE_SPATIAL = 16
LATENT_CHANNELS = 24
PATCH = (1, 2, 2)             # (t, h, w)


def ticks_per_source_frame() -> Fraction:
    """(1/fps) / (1/40 s) clock units."""
    return Fraction(1, VIDEO_FPS) / Fraction(1, AUDIO_LATENT_HZ)


def ticks_per_latent_frame() -> Fraction:
    """A latent frame spans VAE_TEMPORAL_STRIDE source frames."""
    return VAE_TEMPORAL_STRIDE * ticks_per_source_frame()


def latent_frames_per_second() -> Fraction:
    return Fraction(VIDEO_FPS, VAE_TEMPORAL_STRIDE)


def seconds(ticks) -> Fraction:
    return Fraction(ticks) / AUDIO_LATENT_HZ


def causal_latent_count(source_frames: int, stride: int = VAE_TEMPORAL_STRIDE) -> int:
    """(T - 1)/r + 1: the first frame alone makes one latent."""
    if source_frames < 1 or (source_frames - 1) % stride:
        raise ValueError("causal downsampler needs T = 1 + r * k")
    return (source_frames - 1) // stride + 1


def numbers_per_token(channels: int = LATENT_CHANNELS, patch=PATCH) -> int:
    return channels * patch[0] * patch[1] * patch[2]


def tokens_per_latent_frame(latent_h: int, latent_w: int, patch=PATCH) -> int:
    if latent_h % patch[1] or latent_w % patch[2]:
        raise ValueError("latent grid not divisible by the patch")
    return (latent_h // patch[1]) * (latent_w // patch[2])
