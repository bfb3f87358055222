"""Ulysses head sharding through NCCL and the library kernels (world size 1:
the exchanges are identities, so the result must equal the plain path bit for bit)."""
import os
import socket

import numpy as np
import pytest

torch = pytest.importorskip("torch")

import workload as W
from tests.gpu_util import to_dev

pytestmark = pytest.mark.gpu


def test_ulysses_world_one_equals_plain_path():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import torch.distributed as dist
    import packed_mm_rope_b200 as h3
    from packed_mm_rope_b200.ulysses import ulysses_packed_mmrope_attention
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda", 0))
    try:
        wl = W.workload(0)
        perm = W.permutation(wl)
        dperm = torch.from_numpy(perm.astype(np.int32)).cuda()
        q, k, v = (to_dev(a) for a in W.qkv_bf16(wl))
        o_u = ulysses_packed_mmrope_attention(wl.segments, q, k, v, perm=dperm)
        o_p = h3.packed_mmrope_attention(wl.segments, q, k, v, perm=dperm)
        torch.cuda.synchronize()
        assert torch.equal(o_u, o_p)
    finally:
        dist.destroy_process_group()
