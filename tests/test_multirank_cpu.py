"""Host logic of the multi-GPU paths, on CPU with two gloo ranks: in the
benchmark each rank draws its own batch of the same shapes (no data is
exchanged), the timing is the max over ranks, and every rank takes the same
collective steps; when ranks split one batch instead, each rank's slice
(with its rows' whole-sequence positions) gives the unsharded result, and so
does each rank's share of the heads."""
import os
import socket

import numpy as np
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


def _shard_worker(rank, world, port, out):
    """One rank's slice of one batch: the rank runs the oracle on its own rows
    (with their whole-sequence positions) and the slices are gathered."""
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from dit_token_b200 import workloads as W
    from dit_token_b200.shard import shard_packing
    from _util import tbits
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        w = W.custom("sp", (700, 45, 300), (704, 48, 304), hidden=128, num_q_heads=2, num_k_heads=1,
                     head_dim=64, inner=64, grids=((4, 6, 25), (0, 0, 0), (3, 5, 10)), sections=(24, 20, 20))
        inp = W.qk_inputs(w)
        q, k = tbits(W.rows_view(inp["q"])), tbits(W.rows_view(inp["k"]))
        sh = shard_packing(w.cu_seqlens, w.cu_seqlens_padded, w.rope_grid, rank, world)
        qo, ko = oracle.qk_rmsnorm_rope(q[sh.rows], k[sh.rows], tbits(inp["q_weight"]), tbits(inp["k_weight"]),
                                        sh.cu_seqlens, sh.cu_seqlens_padded, num_q_heads=2, num_k_heads=1,
                                        head_dim=64, rope_grid=sh.rope_grid, sections=w.sections,
                                        pos_offset=sh.pos_offset)
        mine = torch.from_numpy(np.concatenate([qo.astype(np.int64), ko.astype(np.int64)], axis=1))
        sizes = [torch.zeros(1, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(sizes, torch.tensor([mine.shape[0]]))
        biggest = int(max(s.item() for s in sizes))
        padded = torch.zeros(biggest, mine.shape[1], dtype=torch.int64)
        padded[: mine.shape[0]] = mine
        parts = [torch.zeros_like(padded) for _ in range(world)]
        dist.all_gather(parts, padded)
        if rank == 0:
            got = np.concatenate([p[: int(n.item())].numpy() for p, n in zip(parts, sizes)])
            fq, fk = oracle.qk_rmsnorm_rope(q, k, tbits(inp["q_weight"]), tbits(inp["k_weight"]), w.cu_seqlens,
                                            w.cu_seqlens_padded, num_q_heads=2, num_k_heads=1, head_dim=64,
                                            rope_grid=w.rope_grid, sections=w.sections)
            want = np.concatenate([fq.astype(np.int64), fk.astype(np.int64)], axis=1)
            valid = w.valid_rows()
            out["equal"] = bool(np.array_equal(got[valid], want[valid]))
            out["rows"] = got.shape[0] == want.shape[0]
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_one_batch_with_global_positions():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_shard_worker, args=(2, port, out), nprocs=2, join=True)
    assert out["rows"] and out["equal"]


def _head_worker(rank, world, port, out):
    """Split by heads instead (the layout after a sequence-to-head
    all-to-all): every rank holds all rows and runs the oracle on its q heads
    and the k head they use; the columns are gathered."""
    import sys
    sys.path.insert(0, ROOT)
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    import oracle
    from dit_token_b200 import workloads as W
    from dit_token_b200.shard import head_range
    from _util import tbits
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        D, Hq, Hk = 64, 4, 2
        w = W.custom("hp", (700, 45, 300), (704, 48, 304), hidden=128, num_q_heads=Hq, num_k_heads=Hk,
                     head_dim=D, inner=64, grids=((4, 6, 25), (0, 0, 0), (3, 5, 10)), sections=(24, 20, 20))
        inp = W.qk_inputs(w)
        q, k = tbits(W.rows_view(inp["q"])), tbits(W.rows_view(inp["k"]))
        wq, wk = tbits(inp["q_weight"]), tbits(inp["k_weight"])
        q0, qc, k0, kc = head_range(Hq, Hk, rank, world)
        qo, ko = oracle.qk_rmsnorm_rope(np.ascontiguousarray(q[:, q0 * D:(q0 + qc) * D]),
                                        np.ascontiguousarray(k[:, k0 * D:(k0 + kc) * D]), wq, wk, w.cu_seqlens,
                                        w.cu_seqlens_padded, num_q_heads=qc, num_k_heads=kc, head_dim=D,
                                        rope_grid=w.rope_grid, sections=w.sections)
        parts_q = [torch.zeros(qo.shape, dtype=torch.int64) for _ in range(world)]
        parts_k = [torch.zeros(ko.shape, dtype=torch.int64) for _ in range(world)]
        dist.all_gather(parts_q, torch.from_numpy(qo.astype(np.int64)))
        dist.all_gather(parts_k, torch.from_numpy(ko.astype(np.int64)))
        if rank == 0:
            fq, fk = oracle.qk_rmsnorm_rope(q, k, wq, wk, w.cu_seqlens, w.cu_seqlens_padded, num_q_heads=Hq,
                                            num_k_heads=Hk, head_dim=D, rope_grid=w.rope_grid,
                                            sections=w.sections)
            out["q"] = bool(np.array_equal(np.concatenate([t.numpy() for t in parts_q], axis=1), fq))
            out["k"] = bool(np.array_equal(np.concatenate([t.numpy() for t in parts_k], axis=1), fk))
    finally:
        dist.destroy_process_group()


def test_two_ranks_split_heads():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_head_worker, args=(2, port, out), nprocs=2, join=True)
    assert out["q"] and out["k"]


def _split_worker(rank, world, port, out):
    """The benchmark's --split leg on CPU: each rank plans its slice of one
    batch, its (fake) device times go through the same max-over-ranks and
    line assembly as on the GPU."""
    import argparse
    import sys
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        lines = {}
        for split in (True, False):
            args = argparse.Namespace(workload="batched_varlen", seed=0, scale=1.0, split=split, steps=5,
                                      warmup=3, e2e_steps=2)
            w, whole, tokens, scaling = bench.plan(args, rank, world)
            slow = 1.0 + rank                      # rank 1 is the slow one
            m = {"elapsed_ms": 10.0 * slow, "step_ms": [2.0 * slow] * 5,
                 "op_ms": {op: [0.5 * slow] * 5 for op in bench.OPS}, "clocks": {"sm_mhz": None},
                 "next_ms": {"gated_residual_adaln": 0.4, "frames_to_u8": 0.6}, "graph_ms": 1.9 * slow,
                 "e2e": (300.0 * slow, 1000, 500), "e2e_steps": 2}
            line = bench.assemble(args, world, w, whole, tokens, scaling, m, torch.device("cpu"))
            lines[split] = (line, w.num_valid, w.num_rows_padded, list(w.pos_offset or ()), whole.num_valid)
        out[rank] = lines
    finally:
        dist.destroy_process_group()


def test_split_leg_json_contract():
    mgr = mp.Manager()
    out = mgr.dict()
    port = _free_port()
    mp.spawn(_split_worker, args=(2, port, out), nprocs=2, join=True)
    (l0, n0, r0, po0, total), (l1, n1, r1, po1, _) = out[0][True], out[1][True]
    assert n0 + n1 == total == 69829            # the slices partition the batch's valid tokens
    assert r0 + r1 == 70144                     # ... and its padded rows
    assert po0 == [0, 0] and po1 == [n0 - 25672, 0, 0]   # rank 1 starts inside sequence 1
    for line in (l0, l1):
        assert line["scaling"] == "strong" and line["n_gpus"] == 2 and line["steps"] == 5
        assert line["config"]["parallelism"].startswith("rows2")
        assert line["config"]["valid_tokens"] == total
        # whole-batch tokens over the slowest rank's time
        assert abs(line["value"] - total * 5 / 0.020) < 1.0
        assert abs(line["e2e"]["value"] - total * 2 / 0.600) < 1.0
        assert line["gpu_launches"] == 4 * 5
    weak0, weak1 = out[0][False][0], out[1][False][0]
    assert weak0["scaling"] == "weak" and weak0["config"]["parallelism"].startswith("dp2")
    assert abs(weak0["value"] - 2 * total * 5 / 0.020) < 1.0 and weak0["value"] == weak1["value"]
