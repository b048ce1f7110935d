"""The N > 1 host path of bench.py on CPU: two gloo ranks, max-over-ranks
timing and whole-job weak-scaling throughput (no GPU, no data-path collective)."""
import os
import socket

import pytest
import torch.distributed as dist
import torch.multiprocessing as mp

import bench


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        elapsed = 10.0 + 5.0 * rank               # rank 1 is the slow one
        m = bench.max_over_ranks(world, elapsed)
        out[rank] = (m, bench.job_throughput(world, 100, 1_000_000, m))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_max_and_throughput():
    world = 2
    mgr = mp.get_context("spawn").Manager()
    out = mgr.dict()
    mp.start_processes(_worker, args=(world, _free_port(), out), nprocs=world, join=True, start_method="spawn")
    assert out[0] == out[1]
    m, value = out[0]
    assert m == 15.0
    assert value == pytest.approx(2 * 100 * 1_000_000 / 15e-3 / 1e9)


def test_single_rank_is_identity():
    assert bench.max_over_ranks(1, 3.5) == 3.5
    assert bench.job_throughput(1, 10, 1e9, 1000.0) == pytest.approx(10.0)


def test_bytes_models():
    # algorithmic bytes per call (every input read once, every output written once)
    assert bench.rms_static_bytes(4096, 4096) == 4096 * 3 * 4096 + 2 * 4096 + 4
    assert bench.ln_static_bytes(4096, 4096) == 4096 * 3 * 4096 + 8 * 4096 + 4
    assert bench.fused_dyn_bytes(64, 2816) == 1_267_456
    assert bench.group_bytes(32768, 4096) == 406_847_488
    assert bench.nvfp4_bytes(8192, 7168, False) == 150_484_996
    assert bench.nvfp4_bytes(8192, 7168, True) == 385_366_020
    # the headline: fused add + RMSNorm + dynamic e4m3 at 65536 x 8192
    assert bench.fused_dyn_bytes(bench.HEAD_M, bench.HEAD_D) == 65536 * (7 * 8192 + 4) + 2 * 8192 == 3_758_374_912
