"""C-ABI checks that need no GPU: the library loads, exports every function
include/h3.h declares, and rejects bad arguments on the host before any launch.
"""
import ctypes
import os
import re

import pytest

import packed_mm_rope_b200 as h3
from packed_mm_rope_b200 import _lib
import workload as W

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _declared_functions():
    src = open(os.path.join(ROOT, "include", "h3.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(h3_[a-z_0-9]+)\s*\(", src)))


def test_every_declared_symbol_is_exported():
    names = _declared_functions()
    assert "h3_packed_attention" in names and len(names) >= 7
    lib = ctypes.CDLL(_lib.LIB_PATH)
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.EXPORTED)
    assert h3.h3_host_workspace_bytes(100, 2) == 4 * 51200 + 1280 + 512
    assert h3.h3_host_workspace_bytes(0, 2) == 0


def test_struct_layouts_match_header():
    assert ctypes.sizeof(_lib.h3_segment) == 9 * 4
    assert ctypes.sizeof(_lib.h3_rope_cfg) == 8 + 6 * 4   # double + 6 int32


def test_status_strings():
    assert h3.status_str(0) == "ok"
    assert "expired" in h3.status_str(h3.H3_ERR_TIMEOUT)
    assert h3.status_str(99) == "unknown status"


def _err(fn, *a, **kw):
    with pytest.raises(h3.H3Error) as e:
        fn(*a, **kw)
    return e.value.status


def test_build_coords_rejects_bad_tables():
    segs = W.workload(0).segments
    # row count mismatch
    assert _err(h3.h3_build_coords, segs, 0, 83, 0x1000) == h3.H3_ERR_INVALID_ARG
    # zero denominator, negative count, unknown kind, bad flag
    for bad in [W.Segment(W.SEG_TEXT, 4, t_den=0), W.Segment(W.SEG_TEXT, -1),
                W.Segment(7, 4), W.Segment(W.SEG_TEXT, 4, flags=8),
                W.Segment(W.SEG_AUDIO, 4, channels=3), W.Segment(W.SEG_VIDEO, 2, 0, 4)]:
        assert _err(h3.h3_build_coords, [bad], 0, max(bad.count, 0), 0x1000) == h3.H3_ERR_INVALID_ARG
    # times outside the exactly representable range
    assert _err(h3.h3_build_coords, [W.Segment(W.SEG_TEXT, 2, t_off_num=1 << 24)], 0, 2,
                0x1000) == h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_build_coords, [W.Segment(W.SEG_VIDEO, 3, 2, 2, 0, 0, 1 << 23, 3)], 0, 12,
                0x1000) == h3.H3_ERR_INVALID_ARG
    # unknown video flag
    assert _err(h3.h3_build_coords, [W.Segment(W.SEG_VIDEO, 1, 2, 2, flags=5)], 0, 4,
                0x1000) == h3.H3_ERR_INVALID_ARG
    # too many segments, NULL output
    assert _err(h3.h3_build_coords, [W.text(1)] * 65, 0, 65, 0x1000) == h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_build_coords, [W.text(3)], 0, 3, 0) == h3.H3_ERR_INVALID_ARG


def test_empty_inputs_are_no_ops():
    h3.h3_build_coords([W.text(0)], 0, 0, 0)
    h3.h3_mmrope_qk(0, 0, 0, 0, 0, 0, 1, 128, h3.rope_cfg())
    h3.h3_packed_attention(0, 0, 0, 0, 0, 1, 0, 1, 128)


def test_rope_rejects_bad_config_and_layout():
    P = 0x10000
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 128, h3.rope_cfg(sections=(32, 48, 46))) == \
        h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 128, h3.rope_cfg(sections=(31, 49, 48))) == \
        h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 128, h3.rope_cfg(theta=1.0)) == h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 128, h3.rope_cfg(pair_layout=2)) == \
        h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 128, h3.rope_cfg(freq_rule=2)) == \
        h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 256,
                h3.rope_cfg(head_dim=256, sections=(64, 96, 96))) == h3.H3_ERR_UNSUPPORTED
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 2, 128, h3.rope_cfg()) == h3.H3_ERR_INVALID_ARG
    assert _err(h3.h3_mmrope_qk, P, P, P, P, P, 4, 1, 132, h3.rope_cfg()) == h3.H3_ERR_UNSUPPORTED
    assert _err(h3.h3_mmrope_qk, P + 8, P, P, P, P, 4, 1, 128, h3.rope_cfg()) == h3.H3_ERR_UNSUPPORTED
    assert _err(h3.h3_mmrope_qk, 0, P, P, P, P, 4, 1, 128, h3.rope_cfg()) == h3.H3_ERR_INVALID_ARG   # q out without q
    assert _err(h3.h3_mmrope_qk, 0, 0, 0, P, P, 4, 1, 128, h3.rope_cfg()) == h3.H3_ERR_INVALID_ARG   # no k


def test_attention_rejects_bad_arguments():
    P = 0x10000
    A = h3.h3_packed_attention
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 128, head_dim=64) == h3.H3_ERR_UNSUPPORTED
    assert _err(A, P, P, P, P, 0, 0, 10, 1, 128) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 10, 0, 128) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 1 << 31, 1, 128) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 10, 2, 128) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 132) == h3.H3_ERR_UNSUPPORTED
    assert _err(A, P, P, P + 4, P, 0, 1, 10, 1, 128) == h3.H3_ERR_UNSUPPORTED
    assert _err(A, P, P, 0, P, 0, 1, 10, 1, 128) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 128, d_rope_cs=P) == h3.H3_ERR_INVALID_ARG     # no cfg
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 128, d_rope_cs=P,
                cfg=h3.rope_cfg(sections=(32, 48, 40))) == h3.H3_ERR_INVALID_ARG
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 128, softmax_scale=float("nan")) == h3.H3_ERR_INVALID_ARG


def test_init_without_a_device_fails_cleanly():
    # no GPU in this process: an error status, nothing launched; shutdown with
    # nothing created is a no-op
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    assert _err(h3.h3_init, 0) in (h3.H3_ERR_CUDA, h3.H3_ERR_INVALID_ARG)
    h3.h3_shutdown()
    assert _lib.load().h3_version() == 101


def test_host_calls_check_the_segment_table_before_queuing_anything():
    # A table that does not add up to n_rows is refused before any copy is
    # queued: the host pointers (never dereferenced) and the missing GPU are
    # not reached, so the status is INVALID_ARG, not a CUDA error.
    P, WORK = 0x10000, 0x100000
    cfg = h3.rope_cfg()
    for segs, n in (([W.text(4)], 5), ([W.Segment(W.SEG_TEXT, 4, t_den=0)], 4), ([W.text(1)] * 65, 65)):
        assert _err(h3.h3_packed_mmrope_attention_host, segs, 0, P, P, P, P, WORK, n, 1, cfg) == \
            h3.H3_ERR_INVALID_ARG
        assert _err(_lib.h3_packed_mmrope_attention_host_noalloc, segs, 0, P, P, P, P, n, 1, cfg) == \
            h3.H3_ERR_INVALID_ARG
    # too many head chunks is also refused up front
    assert _err(h3.h3_packed_mmrope_attention_host, [W.text(4)], 0, P, P, P, P, WORK, 4, 65, cfg, 1) == \
        h3.H3_ERR_UNSUPPORTED


def test_rope_table_rejects_bad_arguments():
    P = 0x10000
    T = h3.h3_rope_cos_sin
    h3.h3_rope_cos_sin(0, 0, h3.rope_cfg(), 0)                                     # empty: no-op
    assert _err(T, P, 4, h3.rope_cfg(sections=(32, 48, 46)), P) == h3.H3_ERR_INVALID_ARG
    assert _err(T, 0, 4, h3.rope_cfg(), P) == h3.H3_ERR_INVALID_ARG
    assert _err(T, P, 4, h3.rope_cfg(), 0) == h3.H3_ERR_INVALID_ARG
    assert _err(T, P, 4, h3.rope_cfg(), P + 8) == h3.H3_ERR_UNSUPPORTED             # table not 16-byte aligned
    assert _err(T, P, 4, h3.rope_cfg(head_dim=256, sections=(64, 96, 96)), P) == h3.H3_ERR_UNSUPPORTED
    A = h3.h3_packed_attention
    assert _err(A, P, P, P, P, 0, 1, 10, 1, 128, d_rope_cs=P + 8, cfg=h3.rope_cfg()) == h3.H3_ERR_UNSUPPORTED
