"""Host logic of the multi-GPU benchmark path, on CPU with two gloo ranks:
each rank draws its own batch of the same shapes (no data is exchanged), the
timing is the max over ranks, and every rank takes the same collective steps."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    import sys
    sys.path.insert(0, ROOT)
    import dataclasses
    import bench
    from dit_token_b200 import workloads as W
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w0 = W.workload("tiny", 0)
        w = dataclasses.replace(w0, seed=bench.data_seed(0, rank))
        x = W.residual_inputs(w)["x"]
        elapsed = 10.0 + rank  # rank 1 is the slow one
        mx = bench.reduce_max(elapsed, torch.device("cpu"))
        world_env = bench.dist_env()
        bench.barrier()
        out[rank] = (mx, w.lengths, float(x.float().nan_to_num().sum()), world_env)
    finally:
        dist.destroy_process_group()


def test_two_ranks_shard_batches_and_take_max_time():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    (m0, l0, s0, e0), (m1, l1, s1, e1) = out[0], out[1]
    assert m0 == m1 == 11.0                 # max over ranks
    assert l0 == l1                         # same shapes on every rank
    assert s0 != s1                         # different data: each rank has its own batch
    assert e0 == (2, 0, 0) and e1 == (2, 1, 1)


def test_single_process_needs_no_process_group():
    import sys
    sys.path.insert(0, ROOT)
    import bench
    assert bench.reduce_max(3.5, torch.device("cpu")) == 3.5
    assert bench.data_seed(5, 0) == 5 and bench.data_seed(5, 1) != 5
