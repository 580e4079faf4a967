"""Two-rank paths on the CPU (gloo): the bench's whole-job reduction, and the
claim that a batch shards across ranks with no exchange -- each rank computes
its own sequences and the union equals the single-process result bit for bit.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

import oracle
import sgmv_inputs as gen
from segmented_gather_gemm_expand_b200.sharding import local_metadata, partition_segments


def free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _init(rank, world, port):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    return dist


def _reduce_worker(rank, world, port, q):
    import torch
    import bench
    dist = _init(rank, world, port)
    try:
        t, b, f, n = bench.reduce_over_ranks(10.0 + rank, 100 * (rank + 1), 7, 3 + rank,
                                             torch.device("cpu"), world)
        q.put((rank, t, b, f, n))
    finally:
        dist.destroy_process_group()


def _shard_worker(rank, world, port, q):
    import torch
    dist = _init(rank, world, port)
    try:
        p = gen.custom(seed=31, lengths=[5, 9, 1, 12, 7, 3], K=16, N=24, H=48, offset=8, num_adapters=3,
                       idx=[2, 0, -1, 1, 2, 0])
        part = partition_segments(p.seq_len, p.lora_idx, world, lora_num=3)[rank]
        s, l, a, rows = local_metadata(p.seq_start, p.seq_len, p.lora_idx, part)
        local = oracle.expand_slice(np.ascontiguousarray(p.x[rows]), p.x_dt, p.calls[0].w, p.w_dt,
                                    np.ascontiguousarray(p.y0[rows]), p.out_dt, s, l, a,
                                    p.calls[0].slice_offset, p.calls[0].slice_size, p.add_inputs)
        # exchange the results once, outside any data path, to check them
        out = [None] * world
        dist.all_gather_object(out, (rows.tolist(), local.tolist()))
        if rank == 0:
            full = p.y0.copy()
            for r_rows, r_local in out:
                if r_rows:
                    full[np.array(r_rows)] = np.array(r_local, dtype=np.uint16)
            q.put(("ok", np.array_equal(full, oracle.run_problem(p))))
    finally:
        dist.destroy_process_group()


def _run(fn, world=2):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = free_port()
    procs = [ctx.Process(target=fn, args=(r, world, port, q)) for r in range(world)]
    for pr in procs:
        pr.start()
    for pr in procs:
        pr.join(timeout=180)
    assert all(pr.exitcode == 0 for pr in procs), [pr.exitcode for pr in procs]
    return [q.get(timeout=10) for _ in range(q.qsize())]


def test_reduce_over_ranks_takes_max_time_and_sums_work():
    res = _run(_reduce_worker)
    assert len(res) == 2
    for rank, t, b, f, n in res:
        assert t == 11.0 and b == 300.0 and f == 14.0 and n == 7.0


def test_sharded_oracle_equals_single_process():
    res = _run(_shard_worker)
    assert res == [("ok", True)]


def test_partition_balances_active_rows():
    L = [100, 5, 5, 300, 1, 1, 90, 200, -3]
    idx = [0, 1, -1, 2, 0, 1, 2, 0, 1]
    parts = partition_segments(L, idx, 3, lora_num=3)
    assert parts[0][0] == 0 and parts[-1][1] == len(L)
    assert all(a[1] == b[0] for a, b in zip(parts, parts[1:]))
    work = [sum(max(L[i], 0) for i in range(*pr) if idx[i] >= 0) for pr in parts]
    assert sum(work) == sum(max(l, 0) for l, i in zip(L, idx) if i >= 0)
    assert max(work) <= 2 * (sum(work) / 3) + 300


def test_partition_edge_cases():
    assert partition_segments([], [], 4) == [(0, 0)] * 4
    assert partition_segments([3], [0], 1) == [(0, 1)]
    with pytest.raises(ValueError):
        partition_segments([3], [0], 0)
