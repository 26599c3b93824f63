"""The N>1 path of bench.py without a GPU: two gloo ranks on this host.

bench.py runs one full batch per rank (weak scaling over independent (b, h)
units: the WKV-7 path has no data-path exchange) and joins the ranks only to
time them: every timing is reduced with a max over ranks, and the job's
throughput is all ranks' tokens over the slowest rank's step.  This test runs
exactly those host-side pieces as two processes over gloo (127.0.0.1) and
checks the reduction, the aggregate and that each rank draws its own batch.
"""
from __future__ import annotations

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, out):
    import bench
    from linear_recurrent_lm_b200 import inputs as I
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        local = [10.0 + 5.0 * rank, 3.0 - rank, 7.5]          # rank 1 slower on the first timing only
        got = bench.rank_max(local, torch.device("cpu"), world)
        wl = I.make_workload(1, seed=bench.rank_seed(rank))
        out[rank] = (got, float(wl.inputs["r"].astype(np.float64).sum()))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_reduce_timings_with_max_and_draw_distinct_batches():
    world, port = 2, _free_port()
    out = mp.get_context("spawn").Manager().dict()
    mp.start_processes(_rank_main, args=(world, port, out), nprocs=world, join=True, start_method="spawn")
    (m0, r0), (m1, r1) = out[0], out[1]
    assert m0 == m1 == [15.0, 3.0, 7.5]        # the slowest rank decides every timing
    assert r0 != r1                           # each rank times its own batch


def test_job_throughput_is_all_ranks_tokens_over_the_slowest_step():
    import bench
    assert bench.job_tokens_per_s(8 * 4096, 1, 2.0) == pytest.approx(8 * 4096 / 2e-3)
    assert bench.job_tokens_per_s(8 * 4096, 4, 2.0) == pytest.approx(4 * 8 * 4096 / 2e-3)
    assert bench.rank_max([1.0, 2.0], torch.device("cpu"), 1) == [1.0, 2.0]
