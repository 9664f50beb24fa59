"""Host-side multi-rank logic of bench.py on CPU: two gloo ranks, each with its
own batch (weak scaling, no data-path collective), time reduced by max over
ranks, whole-job value = units of all ranks / max time."""
import os
import socket

import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world), LOCAL_RANK=str(rank))
    import torch

    import bench

    w, r, local = bench.dist_env()
    assert (w, r) == (world, rank)
    dist = bench.init_dist(world, "gloo")
    dev = torch.device("cpu")
    bench.barrier(dist, dev)
    my_seconds = 1.0 + rank  # rank 1 is the slow one
    tmax = bench.max_over_ranks(my_seconds, dist, dev)
    value = bench.whole_job_value(units_per_rank=64, units_per_step=64, world=world, seconds_max=tmax,
                                  steps=100)
    out[rank] = (tmax, value)
    dist.destroy_process_group()


@pytest.mark.timeout(120)
def test_two_rank_max_and_weak_scaling_value():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True,
                       start_method="spawn")
    for r in range(world):
        tmax, value = out[r]
        assert tmax == 2.0
        # 2 ranks x 100 steps of 64 units in 2 s -> 100 whole-job steps/s
        assert abs(value - 100.0) < 1e-9


def test_step_bytes_counts_scored_and_attended_rows():
    import numpy as np

    import bench
    from head_adaptive_kv_b200.workloads import WORKLOADS

    wl = WORKLOADS[2]
    U = wl.units
    b = bench.step_bytes(wl, np.full(U, 16064), np.full(U, 256), np.full(U, 64), np.full(U, 2048))
    # keys read once with a 4-byte score and a 16-byte logit record written per key
    scored = U * 16064 * (128 * 2 + 4 + 16)
    # dense and condensed K and V; selected tokens: V row and logit record
    attended = U * (256 + 64) * 2 * 128 * 2 + U * 2048 * (128 * 2 + 16)
    assert b - scored - attended == wl.B * wl.Hq * 128 * 2 + wl.B * wl.Hq * 129 * 4 + U * 2048 * 4 + U * 4
