"""The multi-GPU path of the benchmark is independent replicas (streams do not
exchange anything inside the module): each rank runs the same frames on its own
inputs and the job's rate is the units all ranks processed over the slowest
rank's time.  These tests run that host logic as two gloo ranks on the CPU."""
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, ms_per_rank, steps, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        import bench
        value, ms_max = bench.whole_job_rate(ms_per_rank[rank], steps, world, dist, "cpu")
        out[rank] = (value, ms_max)
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_whole_job_rate_takes_slowest_rank():
    world, steps = 2, 40
    ms = [12.5, 20.0]
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_rank_main, args=(world, _free_port(), ms, steps, out), nprocs=world,
                       start_method="spawn", join=True)
    want = steps * world / (max(ms) / 1e3)
    for r in range(world):
        value, ms_max = out[r]
        assert ms_max == max(ms)
        assert value == pytest.approx(want, rel=1e-12)


def test_single_rank_rate_needs_no_process_group():
    import bench
    value, ms_max = bench.whole_job_rate(10.0, 5, 1, None)
    assert ms_max == 10.0 and value == pytest.approx(500.0)


def test_replicas_draw_distinct_inputs():
    """Rank r seeds its stream with an offset of r: replicas must not time the
    same inputs (that would let one rank's caches serve another's)."""
    from hybrid_linear_attention_arl2_b200 import workloads as W
    cfg = W.CONFIGS[1]
    qa = W.Workload(cfg, seed=cfg.seed + 100 * 0).pool_entry(0, 0)[0]
    qb = W.Workload(cfg, seed=cfg.seed + 100 * 1).pool_entry(0, 0)[0]
    assert qa.shape == qb.shape
    assert not np.array_equal(qa, qb)
