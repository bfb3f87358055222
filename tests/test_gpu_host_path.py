"""The host-buffer entry point: same results as the device path, any chunking."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import pipeline as opipe
from tests.gpu_util import bf16_bits_to_f64, check_attention, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def _host(bits, pin):
    t = torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16)
    return t.pin_memory() if pin else t


@pytest.mark.parametrize("cfg,chunk,pin", [(0, 0, True), (1, 0, True), (1, 1, True), (1, 3, False), (1, 8, True)])
def test_host_path_equals_device_path(h3, cfg, chunk, pin):
    wl = W.workload(cfg)
    perm = W.permutation(wl)
    q, k, v = W.qkv_bf16(wl)
    dperm = None if perm is None else torch.from_numpy(perm.astype(np.int32)).cuda()
    o_dev = h3.packed_mmrope_attention(wl.segments, to_dev(q), to_dev(k), to_dev(v), perm=dperm)
    hperm = None if perm is None else torch.from_numpy(perm.astype(np.int32))
    o_host = h3.packed_mmrope_attention_host(wl.segments, _host(q, pin), _host(k, pin), _host(v, pin),
                                             perm=hperm, heads_per_chunk=chunk)
    torch.cuda.current_stream().synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK
    assert torch.equal(o_host, o_dev.cpu())
    if cfg == 0:
        ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v)
        got = bf16_bits_to_f64(o_host.view(torch.int16).numpy().view(np.uint16))
        check_attention(got, ref, "host path")


@pytest.mark.parametrize("heads", [42, 13])
def test_host_path_tapered_chunks_many_heads(h3, heads):
    # the small workload's rows with many heads: the library's own chunking
    # (whole-wave chunks, then the last few heads in halving chunks) must give
    # exactly the device-path result
    import dataclasses
    wl = dataclasses.replace(W.workload(1), heads=heads)
    q, k, v = W.qkv_bf16(wl)
    perm = W.permutation(wl)
    dperm = None if perm is None else torch.from_numpy(perm.astype(np.int32)).cuda()
    o_dev = h3.packed_mmrope_attention(wl.segments, to_dev(q), to_dev(k), to_dev(v), perm=dperm)
    hperm = None if perm is None else torch.from_numpy(perm.astype(np.int32))
    o_host = h3.packed_mmrope_attention_host(wl.segments, _host(q, True), _host(k, True), _host(v, True),
                                             perm=hperm, heads_per_chunk=0)
    torch.cuda.current_stream().synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK
    assert torch.equal(o_host, o_dev.cpu())


def test_host_path_rejects_bad_workspace(h3):
    wl = W.workload(0)
    q, k, v = (_host(a, True) for a in W.qkv_bf16(wl))
    need = h3.h3_host_workspace_bytes(wl.n_rows, wl.heads)
    ws = torch.empty(need + 256, dtype=torch.uint8, device="cuda")
    with pytest.raises(h3.H3Error) as e:
        h3.packed_mmrope_attention_host(wl.segments, q, k, v, perm=torch.zeros(82, dtype=torch.int32),
                                        workspace=ws[8:8 + need])      # large enough, misaligned
    assert e.value.status == h3.H3_ERR_INVALID_ARG
