"""Multi-rank host logic of bench.py on CPU: two gloo ranks in separate processes."""
import os
import socket

import numpy as np
import pytest

import bench
import synth


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import datetime

    import torch
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    try:
        bench.rank_barrier(world)
        local = [1.5, 2.5][rank]  # this rank's "device time"
        t = bench.rank_max(local, world, torch.device("cpu"))
        wl = synth.WORKLOADS["tiny"]
        x = bench.rank_inputs(wl, rank)[synth.TID_X]
        out[rank] = (t, bench.job_tflops(1e12, 4, world, t), x.tobytes())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks():
    import torch.multiprocessing as mp
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    port = _free_port()
    mp.start_processes(_rank_main, args=(2, port, out), nprocs=2, join=True,
                       start_method="spawn")
    (t0, v0, x0), (t1, v1, x1) = out[0], out[1]
    assert t0 == t1 == 2.5              # every rank sees the slowest rank's time
    assert v0 == v1 == 1e12 * 4 * 2 / 2.5 / 1e12  # all ranks' work over that time
    assert x0 != x1                     # own token slice per rank
    wl = synth.WORKLOADS["tiny"]
    a = np.frombuffer(x0, np.uint16)
    assert a.size == wl.linears[0].M * wl.linears[0].K  # same shape on every rank


def test_single_rank_is_identity():
    assert bench.rank_max(3.0, 1, None) == 3.0
    assert bench.job_tflops(2e12, 10, 1, 2.0) == pytest.approx(10.0)
