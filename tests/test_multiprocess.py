"""Multi-rank host logic on CPU (gloo, world size 2).

The recurrence shards over independent (sequence, head) units, so ranks
share no data: each rank draws its own batch (seed = rank) and the only
cross-rank step is the max of the device times.  These tests run that logic
with two gloo ranks on the CPU, with the oracle standing in for the kernel.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, out):
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        import oracle
        import workloads as W
        # every rank draws its own units
        seed = bench.rank_workload_seed(rank)
        inp = W.make_chunk_inputs("kda", "extended", "f32", B=2, T=24, H=2, d_k=8, d_v=4, seed=seed)
        o, sf = oracle.recurrence(inp)
        d_o, _ = W.grad_outputs(inp, seed=seed)          # the backward leg's incoming gradient, per rank
        digest = torch.tensor([float(np.abs(o).sum()), float(np.abs(sf).sum()), float(d_o.abs().sum())],
                              dtype=torch.float64)
        gathered = [torch.zeros(3, dtype=torch.float64) for _ in range(world)]
        dist.all_gather(gathered, digest)
        # max over ranks of a per-rank "device time"
        t = bench.max_over_ranks(0.5 + rank, world)
        out[rank] = (seed, [g.tolist() for g in gathered], t)
    finally:
        dist.destroy_process_group()


def test_two_ranks_own_distinct_units_and_agree_on_slowest_time():
    world = 2
    port = _free_port()
    manager = mp.get_context("spawn").Manager()   # no fork of a process that may hold threads or a CUDA context
    out = manager.dict()
    mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
    seeds = [out[r][0] for r in range(world)]
    assert seeds == [0, 1]
    g0, g1 = out[0][1], out[1][1]
    assert g0 == g1                       # everyone saw the same gathered digests
    assert g0[0] != g0[1]                 # ...and the two ranks' units differ
    assert g0[0][2] != g0[1][2]           # including the backward's incoming gradients
    assert out[0][2] == out[1][2] == 1.5  # max over ranks


def test_rank_seed_is_identity():
    import bench
    assert [bench.rank_workload_seed(r) for r in range(4)] == [0, 1, 2, 3]
