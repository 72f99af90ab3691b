"""Host logic of the multi-rank (weak scaling) bench path on CPU with gloo,
world size 2: every rank gets its own seeded batch of the same shape and the
reported time is the maximum over ranks. No data-path collective exists."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        from moba_inputs import WORKLOADS, make_inputs

        w = WORKLOADS["tiny_fp32"]
        wr = bench.rank_workload(w, rank)
        q, k, v, cu = make_inputs(wr, "cpu")
        t = bench.reduce_max(1.0 + rank, world, "cpu")
        out[rank] = (wr.seed, float(q.sum()), t, wr.lengths == w.lengths)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_batches_and_take_max_time():
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    (s0, q0, t0, same0), (s1, q1, t1, same1) = out[0], out[1]
    assert s0 != s1 and q0 != q1          # independent batches
    assert same0 and same1                # same shapes (weak scaling)
    assert t0 == t1 == 2.0                # slowest rank's time on every rank
