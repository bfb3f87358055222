"""fp64 CPU oracle for packed MM-RoPE attention -- TEST INFRASTRUCTURE ONLY.

Only the test suite, the package smoke check and the benchmark's CPU-baseline
leg may import this package.  The product path (the CUDA library and its
Python binding) never calls it and shares no code with it; the two meet only
at the seeded inputs of the ``workload`` module.

What it computes (plain definitions, fp64 unless stated):

* ``coords``    -- packed segment table -> exact rational (t, h, w) per row,
                   and the correctly rounded fp32 value of each coordinate.
* ``rope``      -- per-axis inverse frequencies and the 2x2 block rotation of
                   Q and K by those coordinates.
* ``attention`` -- exact softmax attention O = softmax(Q K^T / sqrt(D)) V per
                   head over all packed rows (non-causal, no mask).
* ``clock``     -- the time-unit facts the pages state (40 Hz audio ticks,
                   5/3 ticks per 24 fps source frame, 4x temporal stride).
* ``adaln``     -- per-row AdaLN modulation: LayerNorm without its own affine,
                   then (1 + scale[e]) and shift[e] with e = timestep * 3 + tag.

Sources (page titles as published):
  [P1] "Inside MiniMax H3: One DiT Stream for Text, Video, and Stereo Audio"
       (thread; sections 2 "Every modality enters one packed sequence",
       4 "RoPE creates a shared physical timeline", 6 "Long video turns
       attention into the bottleneck").
  [P3] "MiniMax H3 -- one transformer that denoises video and audio together"
       (illustrated explainer; no section numbers, cited by passage).
  [P4] "MiniMax Opens H3 Base Weights: 33B Single-Stream Model ..." (news).
  [P5] "MiniMax H3 -- Open-Weights Omni-Reference Video-Audio Generation Model
       Card" (section "H3-Omni-Transformer").

Every function is pinned by a ``-m "not gpu"`` test against facts the pages
print or against closed forms and invariants; none is "parity unpinned".
"""
from . import adaln, clock, coords, rope, attention  # noqa: F401
from .pipeline import packed_mmrope_attention, rotated_qk  # noqa: F401
