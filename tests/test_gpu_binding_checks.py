"""The Python binding refuses buffers the kernels would read or write out of bounds.

Every case here raises in the binding, before the library is called: a tensor
on the host where the kernels dereference a device pointer, an output or a
workspace too small for the call, a table of the wrong shape.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def _qkv(n, h, seed):
    g = torch.Generator(device="cuda").manual_seed(seed)
    return [torch.randn((n, h, 128), generator=g, device="cuda").to(torch.bfloat16) for _ in range(3)]


def test_coordinate_buffers(h3):
    n = 40
    segs = [W.text(n)]
    with pytest.raises(ValueError):
        h3.build_coords(segs, n, out=torch.empty((n - 1, 3), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        h3.build_coords(segs, n, out=torch.empty((n, 3), dtype=torch.float32))          # host memory
    with pytest.raises(ValueError):
        h3.build_coords(segs, n, perm=torch.arange(n, dtype=torch.int32))               # host memory
    coords = h3.build_coords(segs, n)
    q, k, _ = _qkv(n, 2, 1)
    with pytest.raises(ValueError):
        h3.mmrope_qk(q, k, coords.cpu())
    with pytest.raises(ValueError):
        h3.rope_cos_sin(coords.cpu())
    with pytest.raises(ValueError):
        h3.rope_cos_sin(coords, out=torch.empty((n, 64, 2), dtype=torch.float32))
    torch.cuda.synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK


def test_attention_buffers(h3):
    n, h = 70, 2
    q, k, v = _qkv(n, h, 2)
    with pytest.raises(ValueError):
        h3.packed_attention(q, k, v, lse=torch.empty((1, h, n), dtype=torch.float32))    # host memory
    with pytest.raises(ValueError):
        h3.packed_attention(q, k, v, lse=torch.empty((1, h, n - 1), dtype=torch.float32, device="cuda"))
    with pytest.raises(ValueError):
        h3.packed_attention(q, k, v, rope_cs=torch.zeros((n, 64, 2), dtype=torch.float32))
    with pytest.raises(ValueError):
        h3.packed_attention(q, k, v, out=torch.empty((n - 1, h, 128), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(TypeError):
        h3.packed_attention(q, k, v, out=torch.empty((n, h, 128), dtype=torch.bfloat16))
    torch.cuda.synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK


def test_host_call_buffers(h3):
    wl = W.workload(0)
    q, k, v = (torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
               for a in W.qkv_bf16(wl))
    n, hh = wl.n_rows, wl.heads
    need = h3.h3_host_workspace_bytes(n, hh)
    with pytest.raises(ValueError):
        h3.packed_mmrope_attention_host(wl.segments, q, k, v, out=torch.empty((n - 1, hh, 128), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        h3.packed_mmrope_attention_host(wl.segments, q, k, v, out=q.cuda())
    with pytest.raises(ValueError):
        h3.packed_mmrope_attention_host(wl.segments, q, k, v,
                                        workspace=torch.empty(need - 256, dtype=torch.uint8, device="cuda"))
    with pytest.raises(ValueError):
        h3.packed_mmrope_attention_host(wl.segments, q, k, v, workspace=torch.empty(need, dtype=torch.uint8))
    with pytest.raises(ValueError):
        h3.packed_mmrope_attention_host(wl.segments, q, k, v, perm=torch.zeros(n, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK


def test_adaln_buffers(h3):
    n, c = 5, 64
    x = torch.randn((n, c), device="cuda").to(torch.bfloat16)
    ts = torch.zeros(n, dtype=torch.int32, device="cuda")
    tags = torch.zeros(n, dtype=torch.int32, device="cuda")
    table = torch.zeros((3, 2, c), dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        h3.adaln_modulate(x, ts, tags, table.cpu())
    with pytest.raises(ValueError):
        h3.adaln_modulate(x, ts, tags, table, out=torch.empty((n - 1, c), dtype=torch.bfloat16, device="cuda"))
    with pytest.raises(ValueError):
        h3.adaln_modulate(x, ts, tags, table, out=torch.empty((n, c), dtype=torch.bfloat16))
    with pytest.raises(ValueError):
        h3.adaln_modulate(x, ts.cpu(), tags, table)
    y = h3.adaln_modulate(x, ts, tags, table, eps=1e-6)
    torch.cuda.synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK
    assert not torch.isnan(y).any()
