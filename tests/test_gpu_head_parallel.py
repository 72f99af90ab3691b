"""Head-parallel forward on the GPU path: the head shards that the
all-to-all hands to each rank are independent problems, so the CUDA forward
of every shard reproduces the full forward's heads bit for bit; and the
exchange itself, run as a one-rank NCCL group, returns the full forward."""
import os
import socket

import pytest
import torch
import torch.distributed as dist

import long_context_prefill_block_b200 as moba
from long_context_prefill_block_b200.head_parallel import head_ranges, moba_forward_head_parallel
from moba_inputs import small_case

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("world", [2, 4, 8])
def test_head_shards_reproduce_the_full_forward(world):
    q, k, v, cu = small_case((3000, 1200), 16, 4, 128, 128, 3, dtype=torch.bfloat16, seed=651)
    qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
    full, full_lse = moba.moba_forward(qd, kd, vd, cu, 128, 3, return_lse=True)
    for h0, nh, g0, ng in head_ranges(16, 4, world):
        o, l = moba.moba_forward(qd[:, h0:h0 + nh].contiguous(), kd[:, g0:g0 + ng].contiguous(),
                                 vd[:, g0:g0 + ng].contiguous(), cu, 128, 3, return_lse=True)
        assert torch.equal(o, full[:, h0:h0 + nh])
        assert torch.equal(l, full_lse[:, h0:h0 + nh])
    torch.cuda.synchronize()
    assert moba.moba_device_status() == 0


def test_one_rank_nccl_exchange():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("nccl", rank=0, world_size=1)
    try:
        q, k, v, cu = small_case((2000, 900), 8, 2, 128, 128, 3, dtype=torch.bfloat16, seed=652)
        qd, kd, vd = q.to(DEV), k.to(DEV), v.to(DEV)
        o, l = moba_forward_head_parallel(qd, kd, vd, cu, 128, 3, [q.shape[0]], return_lse=True)
        full, full_lse = moba.moba_forward(qd, kd, vd, cu, 128, 3, return_lse=True)
        torch.cuda.synchronize()
        assert torch.equal(o, full) and torch.equal(l, full_lse)
    finally:
        dist.destroy_process_group()
