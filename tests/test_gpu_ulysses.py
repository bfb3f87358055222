"""Ulysses head sharding through NCCL and the library kernels at world size 1
(one GPU per call here): the exchanges are identities, so the result must
equal the plain path bit for bit, and both must match the fp64 oracle."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from oracle import pipeline as opipe
from tests.gpu_util import bf16_bits_to_f64, check_attention, from_dev_bf16, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def nccl_world_one():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    yield
    dist.destroy_process_group()


@pytest.mark.parametrize("cfg,n_sample", [(0, None), (1, 512)])
def test_ulysses_world_one_matches_oracle_and_plain_path(nccl_world_one, cfg, n_sample):
    import packed_mm_rope_b200 as h3
    from packed_mm_rope_b200.ulysses import ulysses_packed_mmrope_attention
    wl = W.workload(cfg)
    perm = W.permutation(wl)
    dperm = None if perm is None else torch.from_numpy(perm.astype(np.int32)).cuda()
    q, k, v = W.qkv_bf16(wl)
    dq, dk, dv = to_dev(q), to_dev(k), to_dev(v)
    o_u = ulysses_packed_mmrope_attention(wl.segments, dq, dk, dv, perm=dperm)
    o_p = h3.packed_mmrope_attention(wl.segments, dq, dk, dv, perm=dperm)
    torch.cuda.synchronize()
    assert h3.h3_check_device_error() == h3.H3_OK
    assert torch.equal(o_u, o_p)
    rows = None if n_sample is None else W.sample_rows(wl, n_sample)
    ref, _ = opipe.packed_mmrope_attention(wl.segments, perm, q, k, v, wl.theta, wl.sections, rows=rows)
    got = bf16_bits_to_f64(from_dev_bf16(o_u))
    check_attention(got if rows is None else got[rows], ref, f"ulysses {wl.name}")
