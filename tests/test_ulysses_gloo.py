"""Head-sharded (Ulysses) exchange logic on CPU ranks (gloo), uneven splits.

Each rank holds a contiguous shard of the packed rows; the result, gathered
from all ranks, must equal the fp64 oracle on the whole sequence.  The local
per-head attention is the oracle here (the library needs a GPU); the GPU test
runs the library kernels through the same function at world size 1.
"""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _oracle_local(segments, perm, q, k, v, theta, sections, pair_layout):
    from oracle import pipeline
    as_bits = lambda t: t.view(torch.int16).numpy().view(np.uint16)
    o, _ = pipeline.packed_mmrope_attention(segments, perm, as_bits(q), as_bits(k), as_bits(v), theta,
                                            sections, pair_layout=pair_layout)
    # bf16 result of the fp64 values (round to nearest even)
    import workload as W
    return torch.from_numpy(W.bf16_bits_rne(o).view(np.int16)).view(torch.bfloat16)


def _worker(rank, world, port, heads, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    import workload as W
    from packed_mm_rope_b200.ulysses import even_split, ulysses_packed_mmrope_attention
    wl = W.workload(0)                                   # 82 shuffled rows
    perm = W.permutation(wl)
    q, k, v = (W.normal_bf16(321 + i, 0, (wl.n_rows, heads, 128)) for i in range(3))
    rows = even_split(wl.n_rows, world)
    r0 = sum(rows[:rank])
    t = lambda a: torch.from_numpy(a[r0:r0 + rows[rank]].view(np.int16)).view(torch.bfloat16)
    o = ulysses_packed_mmrope_attention(wl.segments, t(q), t(k), t(v), perm=perm,
                                        local_attention=_oracle_local)
    out[rank] = o.view(torch.int16).numpy().copy()
    dist.barrier()
    dist.destroy_process_group()


@pytest.mark.parametrize("world,heads", [(2, 5), (3, 5), (3, 2), (4, 42)])
def test_ulysses_matches_whole_sequence(world, heads):
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), heads, out), nprocs=world, join=True,
                       start_method="spawn")
    got = np.concatenate([out[r] for r in range(world)]).view(np.uint16)
    import workload as W
    from oracle import pipeline
    wl = W.workload(0)
    q, k, v = (W.normal_bf16(321 + i, 0, (wl.n_rows, heads, 128)) for i in range(3))
    ref, _ = pipeline.packed_mmrope_attention(wl.segments, W.permutation(wl), q, k, v)
    np.testing.assert_array_equal(got, W.bf16_bits_rne(ref))


def test_even_split():
    from packed_mm_rope_b200.ulysses import even_split
    assert even_split(42, 4) == [11, 11, 10, 10]      # the pages' 4-GPU deployment of 42 heads
    assert even_split(82, 3) == [28, 27, 27]
    assert even_split(2, 3) == [1, 1, 0]
    with pytest.raises(ValueError):
        even_split(3, 0)
