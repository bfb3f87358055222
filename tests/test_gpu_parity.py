"""GPU parity: the CUDA path through the C ABI against the fp64 oracle.

Coordinates must be bit-exact; rotated Q/K within one bf16 ulp (plus fp32
slack); attention within max |err| <= 2e-2, mean |err| <= 2e-3 and relative
error <= 1e-2 against the oracle on the same bf16 inputs.  Small workloads
are compared in full; the three large ones (28,196 / 81,792 / 31,952 rows x
42 heads) run in full on the GPU in the benchmark's launch configuration and
are compared on >= 2,048 seeded query rows (every segment kind, rows 0 and
N-1, the whole last partial tile, a row in every 256-row block) for all 42
heads.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import attention as oattn
from oracle import coords as ocoords
from oracle import pipeline as opipe
from oracle import rope as orope
from tests.gpu_util import (bf16_bits_to_f64, check_attention, check_rope, from_dev_bf16, to_dev)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def _perm_dev(perm):
    return None if perm is None else torch.from_numpy(perm.astype(np.int32)).cuda()


def _sync_ok(h3):
    st = h3.h3_check_device_error()
    assert st == h3.H3_OK, h3.status_str(st)


# ------------------------------------------------------------ coordinates --

@pytest.mark.parametrize("cfg", range(5))
def test_coords_bit_exact(h3, cfg):
    wl = W.workload(cfg)
    perm = W.permutation(wl)
    got = h3.build_coords(wl.segments, wl.n_rows, _perm_dev(perm)).cpu().numpy()
    _sync_ok(h3)
    num, den = ocoords.packed_coords(wl.segments, perm)
    want = ocoords.to_f32(num, den)
    assert got.dtype == np.float32 and got.shape == want.shape
    assert got.tobytes() == want.tobytes()


def test_coords_flags_and_odd_tables(h3):
    segs = [W.text(5, flags=W.FLAG_TEXT_T_ONLY), W.audio(3, 2, t_off=-7, flags=W.FLAG_AUDIO_CHANNEL_H),
            W.Segment(W.SEG_TEXT, 0), W.video(3, 2, 3, t_off_num=-1), W.audio(4, 1, t_off=100),
            W.Segment(W.SEG_VIDEO, 2, 1, 1, 0, 5, 7, 11), W.Segment(W.SEG_VIDEO, 0, 4, 4)]
    n = sum(s.rows for s in segs)
    perm = W.fisher_yates(n, 99)
    for p in (None, perm):
        got = h3.build_coords(segs, n, _perm_dev(p)).cpu().numpy()
        _sync_ok(h3)
        num, den = ocoords.packed_coords(segs, p)
        assert got.tobytes() == ocoords.to_f32(num, den).tobytes()


def test_coords_reject_out_of_range_perm(h3):
    segs = [W.text(10)]
    perm = np.arange(10, dtype=np.int32)
    perm[3] = 10
    out = h3.build_coords(segs, 10, _perm_dev(perm)).cpu().numpy()
    assert h3.h3_check_device_error() == h3.H3_ERR_DEVICE_INPUT
    assert np.isnan(out[3]).all() and np.isfinite(np.delete(out, 3, axis=0)).all()
    assert h3.h3_check_device_error() == h3.H3_OK      # the word was cleared


# ------------------------------------------------------------------- rope --

def _rope_case(h3, wl, rows=None, pair_layout=0, in_place=False, freq_rule=0):
    perm = W.permutation(wl)
    q, k, _ = W.qkv_bf16(wl)
    coords = h3.build_coords(wl.segments, wl.n_rows, _perm_dev(perm))
    qd, kd = to_dev(q), to_dev(k)
    if in_place:
        qo, ko = h3.mmrope_qk(qd, kd, coords, q_out=qd, k_out=kd, pair_layout=pair_layout, freq_rule=freq_rule)
    else:
        qo, ko = h3.mmrope_qk(qd, kd, coords, pair_layout=pair_layout, freq_rule=freq_rule)
    _sync_ok(h3)
    rows = np.arange(wl.n_rows) if rows is None else rows
    num, den = ocoords.packed_coords(wl.segments, perm)
    ang = orope.angles(ocoords.to_f64(num, den)[rows], wl.theta, wl.sections, freq_rule)
    ang32 = orope.angles(ocoords.to_f32(num, den)[rows].astype(np.float64), wl.theta, wl.sections, freq_rule)
    res = []
    for x_bits, out in ((q, qo), (k, ko)):
        x = bf16_bits_to_f64(x_bits[rows])
        exact = orope.rotate(x, ang, pair_layout)
        got = from_dev_bf16(out)[rows]
        res.append(check_rope(got, exact, x, pair_layout, dang=np.abs(ang32 - ang)))
    return res


@pytest.mark.parametrize("cfg", [0, 1])
def test_rope_parity_full(h3, cfg):
    # the ulp bound (plus fp32 slack near cancellation) is asserted inside check_rope
    for frac_rne, _ in _rope_case(h3, W.workload(cfg)):
        assert frac_rne > 0.99


def test_rope_half_split_and_in_place(h3):
    for frac_rne, _ in _rope_case(h3, W.workload(1), pair_layout=1):
        assert frac_rne > 0.99
    for frac_rne, _ in _rope_case(h3, W.workload(0), in_place=True):
        assert frac_rne > 0.99


@pytest.mark.parametrize("layout", [0, 1])
def test_rope_single_frequency_ladder(h3, layout):
    for frac_rne, _ in _rope_case(h3, W.workload(1), pair_layout=layout, freq_rule=1):
        assert frac_rne > 0.99


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_rope_parity_full_size_sampled(h3, cfg):
    # the three large workloads, rotated in full on the GPU; compared on 2,048
    # seeded rows x all heads (plus every segment's first, middle and last row
    # and the last partial tile).  Workload 4 holds the largest |t| (reference
    # audio at -2000 (c + 1) + j, down to about -6,000): the angle-precision case.
    wl = W.workload(cfg)
    for frac_rne, _ in _rope_case(h3, wl, rows=W.sample_rows(wl, 2048)):
        assert frac_rne > 0.99


# -------------------------------------------------------------- attention --

def _random_bf16(shape, seed, scale=1.0):
    return W.normal_bf16(seed, 0, shape, scale)


@pytest.mark.parametrize("n", [1, 2, 100, 127, 128, 129, 255, 256, 257, 383, 600])
def test_attention_edge_sizes(h3, n):
    H = 2
    q, k, v = (_random_bf16((n, H, 128), 50 + n + 7 * i) for i in range(3))
    lse = torch.empty((1, H, n), dtype=torch.float32, device="cuda")
    o = h3.packed_attention(to_dev(q), to_dev(k), to_dev(v), lse=lse)
    _sync_ok(h3)
    o_ref, lse_ref = oattn.attention(*(bf16_bits_to_f64(a) for a in (q, k, v)))
    check_attention(bf16_bits_to_f64(from_dev_bf16(o)), o_ref, f"n={n}")
    np.testing.assert_allclose(lse.cpu().numpy()[0], lse_ref, rtol=0, atol=2e-3)


def test_attention_batch_and_fused_qkv_stride(h3):
    B, N, H = 2, 300, 3
    qkv = _random_bf16((B, N, 3, H, 128), 77)           # fused projection output layout
    dev = to_dev(qkv)
    q, k, v = dev[:, :, 0], dev[:, :, 1], dev[:, :, 2]
    out = torch.zeros((B, N, 3, H, 128), dtype=torch.bfloat16, device="cuda")
    o = h3.packed_attention(q, k, v, out=out[:, :, 0])
    _sync_ok(h3)
    assert (out[:, :, 1:] == 0).all(), "writes stayed inside the output view"
    x = bf16_bits_to_f64(qkv)
    got = bf16_bits_to_f64(from_dev_bf16(o))
    for b in range(B):
        o_ref, _ = oattn.attention(x[b, :, 0], x[b, :, 1], x[b, :, 2])
        check_attention(got[b], o_ref, f"batch {b}")


@pytest.mark.parametrize("gain,cols", [(6.0, slice(512, 600)), (40.0, slice(512, 600)),
                                       (40.0, slice(64, 128)), (200.0, slice(300, 301))])
def test_attention_running_max_rescale(h3, gain, cols):
    # keys of a later tile (or of the second half of one) are scaled so every
    # row's maximum jumps after the running maximum was set: x6 stays inside the
    # kernel's headroom, x40 and x200 force the rescale (second half, one key)
    N, H = 600, 2
    q = _random_bf16((N, H, 128), 201)
    k = _random_bf16((N, H, 128), 202)
    k[cols] = W.bf16_bits_rne(bf16_bits_to_f64(k[cols]) * gain)
    v = _random_bf16((N, H, 128), 203)
    lse = torch.empty((1, H, N), dtype=torch.float32, device="cuda")
    o = h3.packed_attention(to_dev(q), to_dev(k), to_dev(v), lse=lse)
    _sync_ok(h3)
    o_ref, lse_ref = oattn.attention(*(bf16_bits_to_f64(a) for a in (q, k, v)))
    check_attention(bf16_bits_to_f64(from_dev_bf16(o)), o_ref, f"late max x{gain}")
    np.testing.assert_allclose(lse.cpu().numpy()[0], lse_ref, rtol=1e-5, atol=2e-3)


def test_attention_softmax_scale(h3):
    N, H = 333, 1
    q, k, v = (_random_bf16((N, H, 128), 300 + i) for i in range(3))
    o = h3.packed_attention(to_dev(q), to_dev(k), to_dev(v), softmax_scale=0.25)
    _sync_ok(h3)
    o_ref, _ = oattn.attention(*(bf16_bits_to_f64(a) for a in (q, k, v)), scale=0.25)
    check_attention(bf16_bits_to_f64(from_dev_bf16(o)), o_ref, "scale 0.25")


# --------------------------------------------------------- the whole path --

def _pipeline(h3, wl, q, k, v):
    perm = W.permutation(wl)
    o = h3.packed_mmrope_attention(wl.segments, to_dev(q), to_dev(k), to_dev(v), perm=_perm_dev(perm),
                                   theta=wl.theta, sections=wl.sections)
    _sync_ok(h3)
    return perm, bf16_bits_to_f64(from_dev_bf16(o))


@pytest.mark.parametrize("cfg", [0, 1])
def test_pipeline_parity_full(h3, cfg):
    wl = W.workload(cfg)
    q, k, v = W.qkv_bf16(wl)
    perm, got = _pipeline(h3, wl, q, k, v)
    ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections)
    check_attention(got, ref, wl.name)


def test_pipeline_peaky_queries(h3):
    wl = W.workload(1)
    q, k, v = W.qkv_bf16(wl, q_scale=4.0)
    perm, got = _pipeline(h3, wl, q, k, v)
    ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections)
    # logits ~ N(0, 16): absolute tolerances scale with the logit magnitude (x4)
    check_attention(got, ref, "peaky x4", logit_scale=4.0)


def _rows_covering_every_block(wl, n, block=256):
    """W.sample_rows(wl, n) plus one seeded row in every ``block``-row range, so
    that every (query block, head) CTA of the attention grid has a checked row."""
    N = wl.n_rows
    nb = (N + block - 1) // block
    off = (W.uniform01(wl.seed, 11, nb) * block).astype(np.int64)
    per_block = np.minimum(np.arange(nb, dtype=np.int64) * block + off, N - 1)
    return np.union1d(W.sample_rows(wl, n), per_block)


@pytest.mark.slow
@pytest.mark.parametrize("cfg", [2, 3, 4])
def test_pipeline_parity_full_size_sampled(h3, cfg):
    # the whole path in full on the GPU, in the launch configuration the
    # benchmark times; compared element by element with the fp64 oracle on
    # >= 2,048 seeded query rows x ALL heads (every CTA of the grid covered)
    wl = W.workload(cfg)
    q, k, v = W.qkv_bf16(wl)
    perm, got = _pipeline(h3, wl, q, k, v)
    rows = _rows_covering_every_block(wl, 2048)
    assert rows.size >= 2048
    ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections, rows=rows)
    check_attention(got[rows], ref, wl.name)


def test_row_order_carries_no_position_on_gpu(h3):
    wl = W.workload(0)
    q, k, v = W.qkv_bf16(wl)
    perm, got = _pipeline(h3, wl, q, k, v)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(perm.size)
    o = h3.packed_mmrope_attention(wl.segments, to_dev(q[inv]), to_dev(k[inv]), to_dev(v[inv]))
    _sync_ok(h3)
    unshuffled = bf16_bits_to_f64(from_dev_bf16(o))
    assert np.abs(got - unshuffled[perm]).max() <= 2e-2


# ------------------------------------------- normalised canvas, t-only text --

def test_coords_canvas_bit_exact(h3):
    segs = [W.text(7, flags=W.FLAG_TEXT_T_ONLY), W.video(2, 22, 40, flags=W.FLAG_VIDEO_CANVAS),
            W.video(1, 44, 80, t_off_num=-300, flags=W.FLAG_VIDEO_CANVAS), W.video(3, 9, 16, flags=W.FLAG_VIDEO_CANVAS),
            W.video(2, 5, 3, flags=W.FLAG_VIDEO_CANVAS), W.audio(11, 2)]
    n = sum(s.rows for s in segs)
    perm = W.fisher_yates(n, 123)
    for p in (None, perm):
        got = h3.build_coords(segs, n, _perm_dev(p)).cpu().numpy()
        _sync_ok(h3)
        _, want = ocoords.packed_values(segs, p)
        assert got.tobytes() == want.tobytes()


def test_pipeline_canvas_mode(h3):
    # the pages' own positional scheme: text at (i, 0, 0), video on the canvas
    segs = (W.text(128, flags=W.FLAG_TEXT_T_ONLY), W.video(5, 22, 40, flags=W.FLAG_VIDEO_CANVAS), W.audio(28, 2))
    wl = W.Workload("small_canvas", 1, 8, 128, segs, shuffle=False)
    q, k, v = W.qkv_bf16(wl)
    o = h3.packed_mmrope_attention(segs, to_dev(q), to_dev(k), to_dev(v))
    _sync_ok(h3)
    ref, _ = opipe.packed_mmrope_attention(segs, None, q, k, v)
    check_attention(bf16_bits_to_f64(from_dev_bf16(o)), ref, "canvas")


# -------------------------------------------------- fused RoPE on Q (a5) --

@pytest.mark.parametrize("cfg,layout,rule", [(0, 0, 0), (1, 0, 0), (1, 1, 0), (1, 0, 1), (0, 1, 1)])
def test_fused_q_rope_is_identical_to_rotating_first(h3, cfg, layout, rule):
    wl = W.workload(cfg)
    perm = W.permutation(wl)
    q, k, v = W.qkv_bf16(wl)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    args = dict(perm=_perm_dev(perm), theta=wl.theta, sections=wl.sections, pair_layout=layout, freq_rule=rule)
    o_sep = h3.packed_mmrope_attention(wl.segments, dq, dk, dv, **args)
    o_fus = h3.packed_mmrope_attention(wl.segments, dq, dk, dv, fused_q_rope=True, **args)
    _sync_ok(h3)
    # same rotation arithmetic, same MMAs: bit-identical outputs
    assert torch.equal(o_sep, o_fus)
    ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections, pair_layout=layout,
                                           freq_rule=rule)
    check_attention(bf16_bits_to_f64(from_dev_bf16(o_fus)), ref, f"fused {wl.name}")


@pytest.mark.slow
def test_fused_q_rope_full_size_ref2va(h3):
    # the Ref2VA-shaped workload in full (31,952 rows x 42 heads, reference audio
    # at t down to about -6,000): rotating Q inside the attention kernel from the
    # (cos, sin) table gives exactly the rotate-first output, in every CTA
    wl = W.workload(4)
    perm = W.permutation(wl)
    q, k, v = W.qkv_bf16(wl)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    args = dict(perm=_perm_dev(perm), theta=wl.theta, sections=wl.sections)
    o_sep = h3.packed_mmrope_attention(wl.segments, dq, dk, dv, **args)
    o_fus = h3.packed_mmrope_attention(wl.segments, dq, dk, dv, fused_q_rope=True, **args)
    _sync_ok(h3)
    assert torch.equal(o_sep, o_fus)


@pytest.mark.parametrize("cfg,rule", [(0, 0), (4, 0), (1, 1)])
def test_rope_table_matches_the_oracle_angles(h3, cfg, rule):
    # h3_rope_cos_sin: (cos, sin) of the angle of the fp32 coordinate, each
    # rounded to fp32.  The oracle evaluates the same angle in fp64 with
    # numpy; the two fp64 values differ by a few fp64 ulps at most, so the
    # fp32 results agree except, rarely, by one fp32 ulp at a rounding boundary.
    # Workload 4 holds the largest |t| (reference audio down to about -6,000).
    wl = W.workload(cfg)
    perm = W.permutation(wl)
    coords = h3.build_coords(wl.segments, wl.n_rows, _perm_dev(perm))
    got = h3.rope_cos_sin(coords, theta=wl.theta, sections=wl.sections, freq_rule=rule).cpu().numpy()
    _sync_ok(h3)
    num, den = ocoords.packed_coords(wl.segments, perm)
    ang = orope.angles(ocoords.to_f32(num, den).astype(np.float64), wl.theta, wl.sections, rule)
    want = np.stack([np.cos(ang), np.sin(ang)], axis=-1).astype(np.float32)
    assert got.shape == want.shape == (wl.n_rows, 64, 2)
    ulp = np.spacing(np.abs(want).astype(np.float32))
    assert (np.abs(got.astype(np.float64) - want) <= ulp).all()
    assert (got == want).mean() > 0.9999


def test_rope_k_only_leaves_q_alone(h3):
    wl = W.workload(0)
    perm = W.permutation(wl)
    q, k, _ = W.qkv_bf16(wl)
    coords = h3.build_coords(wl.segments, wl.n_rows, _perm_dev(perm))
    dq, dk = to_dev(q), to_dev(k)
    q_both, k_both = h3.mmrope_qk(dq, dk, coords)
    none, k_only = h3.mmrope_qk(None, dk, coords)
    _sync_ok(h3)
    assert none is None and torch.equal(k_only, k_both)
    assert torch.equal(dq, to_dev(q))


def test_fused_q_rope_ragged_batch(h3):
    B, N, H = 2, 300, 3
    segs = [W.text(20), W.video(2, 10, 12, flags=W.FLAG_VIDEO_CANVAS), W.audio(20, 2)]
    assert sum(s.rows for s in segs) == N
    q, k, v = (W.normal_bf16(400 + i, 0, (B, N, H, 128)) for i in range(3))
    coords = torch.cat([h3.build_coords(segs, N) for _ in range(B)])      # [B*N, 3]
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    qr, kr = h3.mmrope_qk(dq, dk, coords)
    o_sep = h3.packed_attention(qr, kr, dv)
    o_fus = h3.packed_attention(dq, kr, dv, rope_cs=h3.rope_cos_sin(coords))
    _sync_ok(h3)
    assert torch.equal(o_sep, o_fus)


# -------------------------------------------------------------- lifecycle --

def test_init_and_shutdown(h3):
    dev = torch.cuda.current_device()
    h3.h3_init(dev)
    h3.h3_init(dev)                                   # again: harmless
    with pytest.raises(h3.H3Error) as e:
        h3.h3_init(torch.cuda.device_count())
    assert e.value.status == h3.H3_ERR_INVALID_ARG
    assert torch.cuda.current_device() == dev
    # the host-buffer path works, is torn down, and works again after shutdown
    wl = W.workload(0)
    q, k, v = (torch.from_numpy(a.view(np.int16)).view(torch.bfloat16) for a in W.qkv_bf16(wl))
    perm = torch.from_numpy(W.permutation(wl).astype(np.int32))
    o1 = h3.packed_mmrope_attention_host(wl.segments, q, k, v, perm=perm)
    torch.cuda.synchronize()
    h3.h3_shutdown()
    o2 = h3.packed_mmrope_attention_host(wl.segments, q, k, v, perm=perm)
    torch.cuda.synchronize()
    _sync_ok(h3)
    assert torch.equal(o1, o2)
    assert torch.cuda.current_device() == dev


@pytest.mark.parametrize("heads,layout", [(1, 0), (3, 0), (5, 1), (64, 0), (2, 1)])
def test_rope_head_counts(h3, heads, layout):
    # one warp per row, lane l on chunks l, l + 32, ...: head counts that leave
    # lanes idle (1 head = 16 chunks), odd counts, and a wide row
    wl = W.workload(0)
    perm = W.permutation(wl)
    q, k = (W.normal_bf16(500 + heads + i, 0, (wl.n_rows, heads, 128)) for i in range(2))
    coords = h3.build_coords(wl.segments, wl.n_rows, _perm_dev(perm))
    qo, ko = h3.mmrope_qk(to_dev(q), to_dev(k), coords, pair_layout=layout)
    _sync_ok(h3)
    num, den = ocoords.packed_coords(wl.segments, perm)
    ang = orope.angles(ocoords.to_f64(num, den), wl.theta, wl.sections)
    ang32 = orope.angles(ocoords.to_f32(num, den).astype(np.float64), wl.theta, wl.sections)
    for x_bits, out in ((q, qo), (k, ko)):
        x = bf16_bits_to_f64(x_bits)
        frac_rne, _ = check_rope(from_dev_bf16(out), orope.rotate(x, ang, layout), x, layout,
                                 dang=np.abs(ang32 - ang))
        assert frac_rne > 0.99
