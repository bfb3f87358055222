"""GPU parity of h3_adaln_modulate against the fp64 oracle."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import adaln as oadaln
from tests.gpu_util import bf16_bits_to_f64, bf16_ulp, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def h3():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import packed_mm_rope_b200 as lib
    return lib


def _rows_of(wl):
    """Token tag per packed row (0 text, 1 video, 2 audio) and a timestep index:
    conditioning rows (text, single-frame references) at entry 0, the rest at 1."""
    tags, ts = [], []
    for s in wl.segments:
        tags += [s.kind] * s.rows
        ts += [0 if (s.kind == W.SEG_TEXT or (s.kind == W.SEG_VIDEO and s.count == 1)) else 1] * s.rows
    return np.array(ts, np.int32), np.array(tags, np.int32)


@pytest.mark.parametrize("cfg,hidden", [(1, 5376), (0, 128), (4, 5376)])
def test_adaln_matches_oracle(h3, cfg, hidden):
    wl = W.workload(cfg)
    n = wl.n_rows
    x = W.normal_bf16(wl.seed, 9, (n, hidden), scale=2.0)
    ts, tags = _rows_of(wl)
    rng = np.random.default_rng(cfg)
    table = (rng.standard_normal((6, 2, hidden)) * 0.3).astype(np.float32)
    y = h3.adaln_modulate(to_dev(x), torch.from_numpy(ts).cuda(), torch.from_numpy(tags).cuda(),
                          torch.from_numpy(table).cuda())
    assert h3.h3_check_device_error() == h3.H3_OK
    got = bf16_bits_to_f64(from_dev_bf16(y))
    ref = oadaln.adaln_modulate(bf16_bits_to_f64(x), ts, tags, table.astype(np.float64))
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + 1e-5 * (1.0 + np.abs(ref))
    assert (err <= bound).all(), (err.max(), (err > bound).sum())


def test_adaln_in_place_and_bad_index(h3):
    n, c = 50, 256
    x = W.normal_bf16(5, 9, (n, c))
    ts = np.zeros(n, np.int32)
    tags = np.ones(n, np.int32)
    tags[7] = 5                                  # entry 5 does not exist in a 3-entry table
    table = np.random.default_rng(1).standard_normal((3, 2, c)).astype(np.float32)
    dx = to_dev(x)
    out = h3.adaln_modulate(dx, torch.from_numpy(ts).cuda(), torch.from_numpy(tags).cuda(),
                            torch.from_numpy(table).cuda(), out=dx)
    assert h3.h3_check_device_error() == h3.H3_ERR_DEVICE_INPUT
    got = bf16_bits_to_f64(from_dev_bf16(out))
    assert np.isnan(got[7]).all()
    keep = np.delete(np.arange(n), 7)
    ref = oadaln.adaln_modulate(bf16_bits_to_f64(x)[keep], ts[keep], tags[keep], table.astype(np.float64))
    assert (np.abs(got[keep] - ref) <= bf16_ulp(ref) + 1e-5 * (1 + np.abs(ref))).all()


@pytest.mark.parametrize("n,hidden", [(1, 8), (3, 1032), (257, 8192), (130, 4104)])
def test_adaln_widths_and_ragged_row_counts(h3, n, hidden):
    # widths at the chunk boundaries of the kernel (one 16-byte chunk; 129 chunks,
    # one past a whole 128-thread pass; the 8,192 maximum; 513 chunks) and row
    # counts that leave the last row group of a CTA half-used
    x = W.normal_bf16(77 + n, 0, (n, hidden), scale=3.0)
    rng = np.random.default_rng(n)
    ts = rng.integers(0, 2, n).astype(np.int32)
    tags = rng.integers(0, 3, n).astype(np.int32)
    table = (rng.standard_normal((6, 2, hidden)) * 0.3).astype(np.float32)
    y = h3.adaln_modulate(to_dev(x), torch.from_numpy(ts).cuda(), torch.from_numpy(tags).cuda(),
                          torch.from_numpy(table).cuda(), eps=1e-5)
    assert h3.h3_check_device_error() == h3.H3_OK
    got = bf16_bits_to_f64(from_dev_bf16(y))
    ref = oadaln.adaln_modulate(bf16_bits_to_f64(x), ts, tags, table.astype(np.float64), eps=1e-5)
    err = np.abs(got - ref)
    bound = bf16_ulp(ref) + 1e-5 * (1.0 + np.abs(ref))
    assert (err <= bound).all(), (err.max(), (err > bound).sum())


def test_adaln_rejects_unsupported_widths(h3):
    x = torch.zeros((2, 8200), dtype=torch.bfloat16, device="cuda")
    idx = torch.zeros(2, dtype=torch.int32, device="cuda")
    table = torch.zeros((3, 2, 8200), dtype=torch.float32, device="cuda")
    with pytest.raises(h3.H3Error) as e:
        h3.adaln_modulate(x, idx, idx, table)
    assert e.value.status == h3.H3_ERR_UNSUPPORTED
