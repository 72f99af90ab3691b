"""Head-parallel multi-rank forward (token shards in, all-to-all to head
shards with the K/V each rank's heads read, local forward, all-to-all back)
on CPU with gloo. The local forward is the oracle, so the sharded result must
equal the single-process oracle forward bit for bit: every (sequence, head,
query) is computed from the same input bits either way."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from long_context_prefill_block_b200.head_parallel import head_ranges


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _oracle_fn(q, k, v, cu, B, topk, max_seqlen):
    import oracle

    out, lse, _, _ = oracle.forward(q, k, v, cu, B, topk)
    return torch.from_numpy(out), torch.from_numpy(lse)


def _case(seed):
    from moba_inputs import small_case

    return small_case((300, 200, 124), 8, 2, 16, 32, 3, dtype=torch.float32, seed=seed)


def _worker(rank, world, port, shards, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        from long_context_prefill_block_b200.head_parallel import moba_forward_head_parallel

        q, k, v, cu = _case(641)
        a = sum(shards[:rank])
        b = a + shards[rank]
        o, l = moba_forward_head_parallel(q[a:b].contiguous(), k[a:b].contiguous(),
                                          v[a:b].contiguous(), cu, 32, 3, shards,
                                          return_lse=True, forward_fn=_oracle_fn)
        out[rank] = (o.numpy(), l.numpy())
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("shards", [(312, 312), (200, 150, 174, 100)])
def test_head_parallel_equals_single_process(shards):
    import oracle

    world = len(shards)
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), list(shards), out), nprocs=world, join=True)
    q, k, v, cu = _case(641)
    ref, ref_lse, _, _ = oracle.forward(q, k, v, cu, 32, 3)
    got = np.concatenate([out[r][0] for r in range(world)], axis=0)
    got_lse = np.concatenate([out[r][1] for r in range(world)], axis=0)
    assert np.array_equal(got, ref)
    assert np.array_equal(got_lse, ref_lse.astype(np.float32))


def test_head_ranges():
    # whole kv groups per rank, and one kv head shared by (broadcast to) several ranks
    assert head_ranges(8, 2, 2) == [(0, 4, 0, 1), (4, 4, 1, 1)]
    assert head_ranges(8, 2, 4) == [(0, 2, 0, 1), (2, 2, 0, 1), (4, 2, 1, 1), (6, 2, 1, 1)]
    assert head_ranges(32, 8, 4) == [(0, 8, 0, 2), (8, 8, 2, 2), (16, 8, 4, 2), (24, 8, 6, 2)]
    with pytest.raises(ValueError):
        head_ranges(12, 4, 8)  # 12 heads do not split over 8 ranks
    with pytest.raises(ValueError):
        head_ranges(12, 2, 3)  # 4 heads per rank against groups of 6
