"""The allocation-free host-buffer entry point.

Some callers cannot allocate device memory themselves -- for example code
embedded in a host framework that owns the device memory pool, or a
latency-bound loop that must not risk the synchronisation an allocation can
cause.  For them ``h3_packed_mmrope_attention_host_noalloc`` keeps its
workspace in a fixed scratch array inside the library.  These tests call it
through the C ABI and compare it with the workspace variant
``h3_packed_mmrope_attention_host`` on two calls in a row (the scratch keeps
the previous call's contents, so the second call checks that nothing stale
leaks into it), and check that a problem larger than the scratch is refused.
This file is collected last on purpose.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from packed_mm_rope_b200 import _lib
from tests.gpu_util import ATTN_MAX_ABS, ATTN_MEAN_ABS, bf16_bits_to_f64

pytestmark = pytest.mark.gpu


def _pinned(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _as_f64(t):
    return bf16_bits_to_f64(t.view(torch.int16).numpy().view(np.uint16))


def _run_both(wl):
    perm = W.permutation(wl)
    hperm = None if perm is None else torch.from_numpy(perm.astype(np.int32))
    q, k, v = (_pinned(a) for a in W.qkv_bf16(wl))
    cfg = _lib.rope_cfg(wl.theta, 128, wl.sections, 0)
    stream = torch.cuda.current_stream().cuda_stream
    pptr = hperm.data_ptr() if hperm is not None else 0

    o_ref = torch.empty_like(q).pin_memory()
    work = torch.empty(_lib.h3_host_workspace_bytes(wl.n_rows, wl.heads), dtype=torch.uint8, device="cuda")
    _lib.h3_packed_mmrope_attention_host(wl.segments, pptr, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         o_ref.data_ptr(), work.data_ptr(), wl.n_rows, wl.heads, cfg, 0, stream)
    o_new = torch.empty_like(q).pin_memory()
    _lib.h3_packed_mmrope_attention_host_noalloc(wl.segments, pptr, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                 o_new.data_ptr(), wl.n_rows, wl.heads, cfg, stream)
    torch.cuda.current_stream().synchronize()
    assert _lib.h3_check_device_error(stream) == _lib.H3_OK
    return _as_f64(o_new), _as_f64(o_ref)


def test_matches_the_workspace_call_twice_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    # first the small workload (8 heads, 4,584 rows), then the tiny shuffled one
    for idx in (1, 0):
        wl = W.workload(idx)
        assert _lib.h3_host_workspace_bytes(wl.n_rows, wl.heads) <= _lib.H3_NOALLOC_SCRATCH_BYTES
        got, want = _run_both(wl)
        err = np.abs(got - want)
        assert np.isfinite(got).all()
        assert err.max() <= ATTN_MAX_ABS and err.mean() <= ATTN_MEAN_ABS, (idx, err.max(), err.mean())


def test_refuses_problems_larger_than_the_scratch():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    wl = W.workload(2)                       # 28,196 rows x 42 heads needs ~1.2 GB
    assert _lib.h3_host_workspace_bytes(wl.n_rows, wl.heads) > _lib.H3_NOALLOC_SCRATCH_BYTES
    h = torch.empty(16, dtype=torch.uint8)   # never touched: the size check comes first
    cfg = _lib.rope_cfg()
    with pytest.raises(_lib.H3Error) as e:
        _lib.h3_packed_mmrope_attention_host_noalloc(wl.segments, 0, h.data_ptr(), h.data_ptr(), h.data_ptr(),
                                                     h.data_ptr(), wl.n_rows, wl.heads, cfg,
                                                     torch.cuda.current_stream().cuda_stream)
    assert e.value.status == _lib.H3_ERR_TOO_LARGE
