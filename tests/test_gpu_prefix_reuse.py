"""Reuse of the reference rows' keys and values across denoising steps.

"MiniMax H3 -- one transformer ..." (passage on what can be cached): the only
reusable region is block 0's keys and values of the reference rows; every
other row changes at every step.  Since packed row order carries no position,
the reference rows can be placed first in the K/V buffers: their rotated K
and their V are computed once, and each later step rotates and writes only
the fresh rows (a row-range view of the same buffers) before attending over
all rows.  The result must equal recomputing every row.
"""
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import pipeline as opipe
from tests.gpu_util import bf16_bits_to_f64, check_attention, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def test_cached_reference_prefix_equals_full_recompute(h3):
    # reference rows first: 2 images + 1 reference audio clip, then text, target video, target audio
    ref_segs = [W.video(1, 10, 16, t_off_num=-300), W.video(1, 10, 16, t_off_num=-600), W.audio(40, 2, t_off=-2000)]
    fresh_segs = [W.text(64), W.video(4, 10, 16), W.audio(30, 2)]
    segs = ref_segs + fresh_segs
    n_ref = sum(s.rows for s in ref_segs)
    n = sum(s.rows for s in segs)
    H = 4
    coords = h3.build_coords(segs, n)

    # step 1: every row computed; the rotated K and the V of the reference rows are kept
    q1, k1, v1 = (W.normal_bf16(70 + i, 0, (n, H, 128)) for i in range(3))
    kbuf, vbuf = to_dev(k1), to_dev(v1)
    q_rot, _ = h3.mmrope_qk(to_dev(q1), kbuf, coords, k_out=kbuf)       # K rotated in place
    h3.packed_attention(q_rot, kbuf, vbuf)

    # step 2: fresh rows change; reference rows keep their step-1 K, V
    q2, k2, v2 = (W.normal_bf16(80 + i, 0, (n, H, 128)) for i in range(3))
    k2[:n_ref], v2[:n_ref] = k1[:n_ref], v1[:n_ref]
    kbuf[n_ref:] = to_dev(k2[n_ref:])
    vbuf[n_ref:] = to_dev(v2[n_ref:])
    _, _ = h3.mmrope_qk(None, kbuf[n_ref:], coords[n_ref:], k_out=kbuf[n_ref:])   # only the fresh rows
    _, q2_rot = h3.mmrope_qk(None, to_dev(q2), coords)          # all queries are fresh (same rotation)
    o_cached = h3.packed_attention(q2_rot, kbuf, vbuf)

    # reference: recompute every row of step 2 from scratch
    o_full = h3.packed_mmrope_attention(segs, to_dev(q2), to_dev(k2), to_dev(v2))
    assert h3.h3_check_device_error() == h3.H3_OK
    assert torch.equal(o_cached, o_full)
    ref, _ = opipe.packed_mmrope_attention(segs, None, q2, k2, v2)
    check_attention(bf16_bits_to_f64(from_dev_bf16(o_cached)), ref, "cached prefix")
