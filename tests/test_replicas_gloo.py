"""The multi-GPU path on CPU: two gloo ranks, no GPU.

bench.py --gpus N runs one replica of the workload per rank (weak scaling, no
collective on the data path); its only collectives are the barrier and the
max-over-ranks reduction of the timed region. These tests run those helpers on
two real processes: each rank scans its own seeded replica (with the oracle,
standing in for the device here), the replicas must be independent and equal to
a single-process computation, and the job time must be the slowest rank's.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp

from conftest import ROOT


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out_dir):
    import sys
    sys.path.insert(0, ROOT)
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    import workloads

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        assert bench.dist_env() == (world, rank, rank)
        wl = workloads.WORKLOADS["evmamba_atrous_55x57"].with_(batch=1, D=4, h=7, w=9)
        x = workloads.draw(bench.replica(wl, rank))
        y = oracle.forward(wl.route, wl.h, wl.w, x["u"], x["delta"], x["A"], x["B"], x["C"],
                           x["Dskip"], x["bias"], x["z"])
        np.save(os.path.join(out_dir, f"y{rank}.npy"), y)
        # a fake per-rank time: rank r took 10 + r ms
        t = bench.max_over_ranks(10.0 + rank)
        with open(os.path.join(out_dir, f"t{rank}.txt"), "w") as f:
            f.write(repr(t))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_replica_ranks_on_gloo(tmp_path):
    world = 2
    port = _free_port()
    mp.start_processes(_rank_main, args=(world, port, str(tmp_path)), nprocs=world, join=True,
                       start_method="spawn")
    import sys
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    import workloads

    times = [float(open(tmp_path / f"t{r}.txt").read()) for r in range(world)]
    assert times == [11.0, 11.0]
    wl = workloads.WORKLOADS["evmamba_atrous_55x57"].with_(batch=1, D=4, h=7, w=9)
    ys = [np.load(tmp_path / f"y{r}.npy") for r in range(world)]
    assert not np.array_equal(ys[0], ys[1])  # each rank has its own data
    for r in range(world):
        x = workloads.draw(bench.replica(wl, r))
        ref = oracle.forward(wl.route, wl.h, wl.w, x["u"], x["delta"], x["A"], x["B"], x["C"],
                             x["Dskip"], x["bias"], x["z"])
        np.testing.assert_array_equal(ys[r], ref)
    # whole-job throughput: both ranks' units over the slowest rank's time
    units = wl.token_channels
    assert bench.job_throughput(units, 5, world, times[0]) == pytest.approx(units * 5 * 2 / 0.011)
