"""The allocation-free host-buffer entry point.

Some callers cannot allocate device memory themselves -- for example code
embedded in a host framework that owns the device memory pool, or a
latency-bound loop that must not risk the synchronisation an allocation can
cause.  For them ``h3_packed_mmrope_attention_host_noalloc`` keeps its
workspace in a fixed scratch array inside the library.  These tests call it
through the C ABI several times in a row and compare each result with the
workspace variant ``h3_packed_mmrope_attention_host`` on the same inputs.
Both run the same kernels on the same values, so the outputs must be
identical bit for bit.  The scratch keeps the previous call's contents, so
a second call of the same shape with other inputs would show any stale value
that leaked into it; the first result is also checked against the fp64
oracle, and a problem larger than the scratch must be refused.
This file is collected last on purpose.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import pipeline as opipe
from packed_mm_rope_b200 import _lib
from tests.gpu_util import bf16_bits_to_f64, check_attention

pytestmark = pytest.mark.gpu


def _pinned(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).pin_memory()


def _bits(t):
    return t.view(torch.int16).numpy().view(np.uint16)


def _run_both(wl, q_bits, k_bits, v_bits):
    perm = W.permutation(wl)
    hperm = None if perm is None else torch.from_numpy(perm.astype(np.int32))
    q, k, v = (_pinned(a) for a in (q_bits, k_bits, v_bits))
    cfg = _lib.rope_cfg(wl.theta, 128, wl.sections, 0)
    stream = torch.cuda.current_stream().cuda_stream
    pptr = hperm.data_ptr() if hperm is not None else 0

    o_ref = torch.empty_like(q).pin_memory()
    work = torch.empty(_lib.h3_host_workspace_bytes(wl.n_rows, wl.heads), dtype=torch.uint8, device="cuda")
    _lib.h3_packed_mmrope_attention_host(wl.segments, pptr, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                         o_ref.data_ptr(), work.data_ptr(), wl.n_rows, wl.heads, cfg, 0, stream)
    o_new = torch.empty_like(q).pin_memory()
    o_new.fill_(float("nan"))
    _lib.h3_packed_mmrope_attention_host_noalloc(wl.segments, pptr, q.data_ptr(), k.data_ptr(), v.data_ptr(),
                                                 o_new.data_ptr(), wl.n_rows, wl.heads, cfg, stream)
    torch.cuda.current_stream().synchronize()
    assert _lib.h3_check_device_error(stream) == _lib.H3_OK
    return o_new, o_ref


def test_matches_the_workspace_call_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    small = W.workload(1)                    # 4,584 rows x 8 heads
    assert _lib.h3_host_workspace_bytes(small.n_rows, small.heads) <= _lib.H3_NOALLOC_SCRATCH_BYTES
    shape = (small.n_rows, small.heads, 128)
    q, k, v = W.qkv_bf16(small)
    # 1: the small workload, also checked against the fp64 oracle
    got, want = _run_both(small, q, k, v)
    assert torch.equal(got, want)
    ref, _ = opipe.packed_mmrope_attention(small.segments, W.permutation(small), q, k, v, small.theta,
                                           small.sections)
    check_attention(bf16_bits_to_f64(_bits(got)), ref, "no-alloc call")
    # 2: the same shape with other inputs: stale scratch contents would show
    q2, k2, v2 = (W.normal_bf16(4242 + i, 0, shape) for i in range(3))
    got2, want2 = _run_both(small, q2, k2, v2)
    assert torch.equal(got2, want2)
    assert not torch.equal(got2, got)
    # 3: the tiny shuffled workload (row permutation copied in as well)
    tiny = W.workload(0)
    got3, want3 = _run_both(tiny, *W.qkv_bf16(tiny))
    assert torch.equal(got3, want3)


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
