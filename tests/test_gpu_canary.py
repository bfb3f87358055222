"""Out-of-bounds write checks without a sanitizer: canary-filled guard regions.

Every output buffer sits inside a larger allocation filled with a bf16 NaN
payload (0x7FC1) that no kernel produces: guard rows before and after the
tensor, and padding columns at the end of every row (row_stride > H * 128).
After each call the guards must be intact, and the inputs unchanged.  Sizes
are ragged (the last 128-row tile is partial) so the tail handling of every
kernel is exercised.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W

pytestmark = pytest.mark.gpu

CANARY = 0x7FC1          # a NaN payload; kernels write 0x7FC0 for NaN
GUARD_ROWS = 3


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


class Guarded:
    """A [n, h, 128] bf16 view with row stride rs inside a canary-filled buffer."""

    def __init__(self, n, h, pad, fill=None):
        self.n, self.h, self.rs = n, h, h * 128 + pad
        total = (n + 2 * GUARD_ROWS) * self.rs
        self.buf = torch.full((total,), CANARY, dtype=torch.int16, device="cuda")
        self.view = self.buf.view(torch.bfloat16).as_strided((n, h, 128), (self.rs, 128, 1),
                                                              GUARD_ROWS * self.rs)
        if fill is not None:
            self.view.copy_(fill)
        self.snapshot = self.buf.clone()

    def guards_intact(self):
        b = self.buf.view(-1, self.rs)
        g = GUARD_ROWS
        ok = bool((b[:g] == CANARY).all()) and bool((b[g + self.n:] == CANARY).all())
        return ok and bool((b[g:g + self.n, self.h * 128:] == CANARY).all())

    def unchanged(self):
        return torch.equal(self.buf, self.snapshot)


def _rand(n, h, seed):
    bits = W.normal_bf16(seed, 0, (n, h, 128))
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).cuda()


@pytest.mark.parametrize("n", [1, 129, 257])
def test_attention_writes_only_its_output(h3, n):
    H, pad = 3, 8
    q, k, v = (Guarded(n, H, pad, _rand(n, H, 900 + i)) for i in range(3))
    o = Guarded(n, H, pad)
    lse = torch.full((GUARD_ROWS * 2 + H * n,), float("nan"), dtype=torch.float32, device="cuda")
    lse_view = lse[GUARD_ROWS:GUARD_ROWS + H * n].view(1, H, n)
    h3.packed_attention(q.view, k.view, v.view, out=o.view, lse=lse_view)
    assert h3.h3_check_device_error() == h3.H3_OK
    assert o.guards_intact()
    assert all(t.unchanged() for t in (q, k, v))
    assert not torch.isnan(o.view).any() and not torch.isnan(lse_view).any()
    assert torch.isnan(lse[:GUARD_ROWS]).all() and torch.isnan(lse[GUARD_ROWS + H * n:]).all()
    # the same values as a contiguous call
    ref = h3.packed_attention(q.view.contiguous(), k.view.contiguous(), v.view.contiguous())
    assert torch.equal(ref, o.view)


@pytest.mark.parametrize("n", [1, 7, 129])
def test_rope_writes_only_its_outputs(h3, n):
    H, pad = 2, 16
    segs = [W.text(n)]
    coords_buf = torch.full((3 * (n + 2 * GUARD_ROWS),), float("nan"), dtype=torch.float32, device="cuda")
    coords = coords_buf[3 * GUARD_ROWS:3 * (GUARD_ROWS + n)].view(n, 3)
    h3.build_coords(segs, n, out=coords)
    assert torch.isnan(coords_buf[:3 * GUARD_ROWS]).all() and torch.isnan(coords_buf[3 * (GUARD_ROWS + n):]).all()
    assert not torch.isnan(coords).any()
    q, k = Guarded(n, H, pad, _rand(n, H, 950)), Guarded(n, H, pad, _rand(n, H, 951))
    qo, ko = Guarded(n, H, pad), Guarded(n, H, pad)
    h3.mmrope_qk(q.view, k.view, coords, q_out=qo.view, k_out=ko.view)
    assert h3.h3_check_device_error() == h3.H3_OK
    assert qo.guards_intact() and ko.guards_intact()
    assert q.unchanged() and k.unchanged()
    # in place: only the tensor itself changes
    h3.mmrope_qk(q.view, k.view, coords, q_out=q.view, k_out=k.view)
    assert q.guards_intact() and k.guards_intact()
    assert torch.equal(q.view, qo.view) and torch.equal(k.view, ko.view)


def test_adaln_writes_only_its_rows(h3):
    n, c, pad = 37, 5376, 8
    rs = c + pad
    buf = torch.full(((n + 2 * GUARD_ROWS) * rs,), CANARY, dtype=torch.int16, device="cuda")
    y = buf.view(torch.bfloat16).as_strided((n, c), (rs, 1), GUARD_ROWS * rs)
    x = torch.from_numpy(W.normal_bf16(960, 0, (n, c)).view(np.int16)).view(torch.bfloat16).cuda()
    x0 = x.clone()
    ts = torch.zeros(n, dtype=torch.int32, device="cuda")
    tags = (torch.arange(n, dtype=torch.int32, device="cuda") % 3).contiguous()
    table = torch.randn((3, 2, c), dtype=torch.float32, device="cuda")
    h3.adaln_modulate(x, ts, tags, table, out=y)
    assert h3.h3_check_device_error() == h3.H3_OK
    b = buf.view(-1, rs)
    assert (b[:GUARD_ROWS] == CANARY).all() and (b[GUARD_ROWS + n:] == CANARY).all()
    assert (b[GUARD_ROWS:GUARD_ROWS + n, c:] == CANARY).all()
    assert torch.equal(x, x0) and not torch.isnan(y).any()
