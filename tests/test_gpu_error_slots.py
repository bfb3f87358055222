"""Device faults are reported per stream.

Every kernel records a fault in the error word of the stream it was launched
on, and h3_check_device_error(stream) takes only that stream's word.  So a
check of one stream neither reports nor clears a fault raised on another,
and two host threads may check their own streams concurrently.  Faults are
made without touching the GPU's health: a bounded wait forced to expire, and
a permutation entry out of range (both turn into an error status, the kernel
returns normally).
"""
import threading

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def test_timeout_is_reported_only_on_its_own_stream(h3):
    N, H = 1500, 2
    dq, dk, dv = (to_dev(W.normal_bf16(910 + i, 0, (N, H, 128))) for i in range(3))
    segs = [W.text(N)]
    sa, sb = torch.cuda.Stream(), torch.cuda.Stream()
    torch.cuda.synchronize()
    for s in (sa, sb):
        assert h3.h3_check_device_error(s.cuda_stream) == h3.H3_OK
    try:
        h3.h3_set_wait_limit_ns(1)
        h3.packed_attention(dq, dk, dv, stream=sa)          # every wait gives up
        sa.synchronize()                                    # the faulting kernel has finished
        # stream B runs kernels without waits; its check must neither report
        # nor clear stream A's fault
        coords = torch.empty((N, 3), dtype=torch.float32, device="cuda")
        h3.build_coords(segs, N, out=coords, stream=sb)
        h3.mmrope_qk(dq, dk, coords, stream=sb)
        assert h3.h3_check_device_error(sb.cuda_stream) == h3.H3_OK
        assert h3.h3_check_device_error(sa.cuda_stream) == h3.H3_ERR_TIMEOUT
    finally:
        h3.h3_set_wait_limit_ns(0)
    assert h3.h3_check_device_error(sa.cuda_stream) == h3.H3_OK     # taken and cleared once


def test_two_threads_check_their_own_streams(h3):
    from packed_mm_rope_b200 import _lib
    n = 4096
    segs = [W.text(n)]
    good = torch.arange(n, dtype=torch.int32, device="cuda")
    bad = good.clone()
    bad[n // 2] = n                                          # out of range: DEVICE_INPUT
    outs = [torch.empty((n, 3), dtype=torch.float32, device="cuda") for _ in range(2)]
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    torch.cuda.synchronize()
    for s in streams:
        _lib.h3_check_device_error(s.cuda_stream)
    results = [[], []]

    def worker(i):
        s = streams[i].cuda_stream
        perm = bad if i == 0 else good
        for _ in range(25):
            _lib.h3_build_coords(segs, perm.data_ptr(), n, outs[i].data_ptr(), s)
            results[i].append(_lib.h3_check_device_error(s))

    threads = [threading.Thread(target=worker, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert results[0] == [h3.H3_ERR_DEVICE_INPUT] * 25
    assert results[1] == [h3.H3_OK] * 25
    assert np.isnan(outs[0][n // 2].cpu().numpy()).all()
    assert torch.isfinite(outs[1]).all()
