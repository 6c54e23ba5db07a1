"""The multi-GPU path's host logic, on two gloo ranks on the CPU.

Samples are independent, so each rank runs its own batch (weak scaling) and
the only collective is the MAX of the timed duration.  Here: ranks draw
different batches, each rank's result depends only on its own batch, and the
reduction and the whole-job throughput are right.
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


def _rank_main(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import bench
        import oracle
        from workloads import make_workload
        w = make_workload(2, B=3, seed=bench.rank_seed(2, rank))
        o, _ = oracle.forward_workload(w)
        # the shard alone determines the rank's result
        o2, _ = oracle.forward_workload(make_workload(2, B=3, seed=bench.rank_seed(2, rank)))
        lens = [None] * world
        dist.all_gather_object(lens, w.q_lens.tolist())
        t = bench.max_over_ranks(10.0 + rank, torch.device("cpu"))
        out[rank] = dict(same=bool(np.array_equal(o, o2)), lens=lens, t=t,
                         value=bench.job_tflops(2e12, world, t))
    finally:
        dist.destroy_process_group()


def test_two_rank_weak_scaling_logic():
    port = _free_port()
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True,
                       start_method="spawn")
    assert out[0]["same"] and out[1]["same"]
    assert out[0]["lens"] == out[1]["lens"]                 # both ranks saw the same gather
    assert out[0]["lens"][0] != out[0]["lens"][1]           # ...of different batches
    assert out[0]["t"] == out[1]["t"] == 11.0               # max over ranks
    assert out[0]["value"] == pytest.approx(2e12 * 2 / 11e-3 / 1e12)
