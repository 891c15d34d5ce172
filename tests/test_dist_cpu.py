"""Multi-process host logic of bench.py on CPU (gloo, world size 2): ranks are independent
replicas; the job's step time is the slowest rank's and its work is the sum of all ranks'."""
import os
import socket
import sys

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
    sys.path.insert(0, ROOT)
    import bench

    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world),
                      LOCAL_RANK=str(rank))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    assert bench.dist_env() == (world, rank, rank)

    def rmax(v):
        t = torch.tensor([v], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        return float(t.item())

    def rsum(v):
        t = torch.tensor([v], dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        return float(t.item())

    ms_local = 1.0 + rank            # rank 1 is the slow one
    flops_local = 1e12
    ms, flops, tflops = bench.aggregate(ms_local, flops_local, world, rmax, rsum)
    out[rank] = (ms, flops, tflops)
    dist.barrier()
    dist.destroy_process_group()


def test_replicas_aggregate_max_time_and_total_work():
    world = 2
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, _free_port(), out), nprocs=world, join=True)
    for r in range(world):
        ms, flops, tflops = out[r]
        assert ms == 2.0 and flops == 2e12
        assert tflops == pytest.approx(2e12 / 2e-3 / 1e12)


def test_single_process_aggregate_is_identity():
    sys.path.insert(0, ROOT)
    import bench

    ms, flops, tflops = bench.aggregate(0.5, 1e12, 1, float, float)
    assert (ms, flops) == (0.5, 1e12) and tflops == pytest.approx(2000.0)


def test_reference_arm_config_matches_native():
    sys.path.insert(0, ROOT)
    import bench
    from exact_io_aware_68_b200.workloads import WORKLOADS, HEADLINE

    w = WORKLOADS[HEADLINE]
    c = bench.config_of(w, 1)
    assert c["workload"] == HEADLINE and c["N"] == 4096 and c["d"] == 128 and c["causal"]
    assert w.fwd_flops() == pytest.approx(137.4e9, rel=1e-3)
    assert w.fwd_bwd_flops() == pytest.approx(481.0e9, rel=1e-3)
