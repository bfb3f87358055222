"""Per-row AdaLN modulation (fp64).

Definition followed:
* [P3] AdaLN passage: a normalisation with computed (not constant) scale and
  shift, y = norm(x) * (1 + scale) + shift; H3 builds a table indexed by
  (noise level, modality) and every row looks up its own entry,
  ``adaln_indices = timestep_indices * 3 + token_tags``.
* [P1] section 5: shift, scale and gate are selected by the diffusion
  timestep and by whether the row is text, video or audio, computed on a small
  table of unique (timestep, modality) pairs and gathered per row.

Readings (the pages are silent): norm is LayerNorm over the hidden dimension
without its own affine parameters, (x - mean) / sqrt(var + eps) with the
biased variance and eps = 1e-6; token tags 0 = text, 1 = video, 2 = audio;
the table holds (shift, scale) per entry.
"""
from __future__ import annotations

import numpy as np

TAG_TEXT, TAG_VIDEO, TAG_AUDIO = 0, 1, 2


def adaln_index(timestep_index, token_tag):
    """Entry of the modulation table for each row."""
    return np.asarray(timestep_index, np.int64) * 3 + np.asarray(token_tag, np.int64)


def layer_norm(x: np.ndarray, eps: float = 1e-6) -> np.ndarray:
    x = np.asarray(x, np.float64)
    mean = x.mean(axis=-1, keepdims=True)
    var = ((x - mean) ** 2).mean(axis=-1, keepdims=True)
    return (x - mean) / np.sqrt(var + eps)


def adaln_modulate(x, timestep_index, token_tag, table, eps: float = 1e-6):
    """x [N, C]; table [E, 2, C] with [:, 0] = shift, [:, 1] = scale -> y [N, C]."""
    table = np.asarray(table, np.float64)
    e = adaln_index(timestep_index, token_tag)
    if (e < 0).any() or (e >= table.shape[0]).any():
        raise IndexError("modulation index outside the table")
    shift, scale = table[e, 0], table[e, 1]
    return layer_norm(x, eps) * (1.0 + scale) + shift
