"""Failure detection on the GPU without a fault: every mbarrier wait inside the
attention kernel is bounded by device global time.  With the limit forced to
1 ns the waits give up, the kernel drains its own copies and MMAs, frees tensor
memory and returns; the host reads H3_ERR_TIMEOUT from the error word, and the
next call on the same context computes correct results again.
"""
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import attention as oattn
from tests.gpu_util import bf16_bits_to_f64, check_attention, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu


def test_forced_wait_timeout_is_reported_and_context_survives():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as h3
    N, H = 1500, 3
    q, k, v = (W.normal_bf16(900 + i, 0, (N, H, 128)) for i in range(3))
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    assert h3.h3_check_device_error() == h3.H3_OK
    try:
        h3.h3_set_wait_limit_ns(1)
        h3.packed_attention(dq, dk, dv)
        assert h3.h3_check_device_error() == h3.H3_ERR_TIMEOUT
    finally:
        h3.h3_set_wait_limit_ns(0)          # back to the default limit
    assert h3.h3_check_device_error() == h3.H3_OK
    o = h3.packed_attention(dq, dk, dv)
    assert h3.h3_check_device_error() == h3.H3_OK
    ref, _ = oattn.attention(*(bf16_bits_to_f64(a) for a in (q, k, v)))
    check_attention(bf16_bits_to_f64(from_dev_bf16(o)), ref, "after timeout")
