"""The multi-GPU path of bench.py is replicas only (one independent layer per rank, no data-path
collective); its host logic - slowest-rank step time, whole-job value - checked with two gloo
ranks on the CPU."""
import os
import socket

import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    import bench
    from mxfp8_quantize_b200 import workloads
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms_local = [10.0, 12.5][rank]              # rank 1 is the slower replica
        ms = bench.max_over_ranks(ms_local, world)
        cfg = workloads.CONFIGS["mixtral_mxfp8"]
        out[rank] = (ms, bench.job_tflops(cfg, ms, world))
    finally:
        dist.destroy_process_group()


def test_two_replicas_take_the_slowest_rank_and_sum_the_work():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, start_method="spawn")
    from mxfp8_quantize_b200 import workloads
    cfg = workloads.CONFIGS["mixtral_mxfp8"]
    for rank in range(world):
        ms, tf = out[rank]
        assert ms == 12.5
        assert tf == pytest.approx(2 * cfg.flops_fwd_bwd() / 12.5e-3 / 1e12)


def test_single_rank_needs_no_process_group():
    import bench
    assert bench.max_over_ranks(3.0, 1) == 3.0
