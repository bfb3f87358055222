"""The N>1 bench path on CPU: two gloo ranks, barrier + max-over-ranks timing."""
import os
import socket

import pytest

torch = pytest.importorskip("torch")
import torch.distributed as dist  # noqa: E402
import torch.multiprocessing as mp  # noqa: E402


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    from packed_mm_rope_b200 import dist as hdist
    w, r, lr = hdist.world_from_env()
    assert (w, r, lr) == (world, rank, rank)
    hdist.init("gloo", timeout_s=60)
    hdist.barrier()
    t = 10.0 + 5.0 * rank                        # rank 1 is the slow one
    m = hdist.max_over_ranks(t)
    out[rank] = hdist.weak_scaling_throughput(1.0e12, world, m)
    hdist.barrier()
    dist.destroy_process_group()


def test_two_rank_max_and_weak_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    # both ranks see the slowest time (15 s) and count both ranks' work
    assert out[0] == out[1] == pytest.approx(2.0e12 / 15.0)


def test_single_process_fallbacks():
    from packed_mm_rope_b200 import dist as hdist
    assert hdist.max_over_ranks(3.5) == 3.5
    with pytest.raises(ValueError):
        hdist.weak_scaling_throughput(1.0, 1, 0.0)
