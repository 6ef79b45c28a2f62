"""Host logic of the multi-GPU benchmark path, run as two gloo ranks on the CPU.

bench.py --gpus N runs independent replicas (the layer needs no collective); the only
cross-rank steps are the max-over-ranks reduction of the timed region and the whole-job
throughput. These tests check both with world_size 2 without a GPU.
"""
import os
import socket

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
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = 10.0 + 7.5 * rank  # rank 1 is the slow one
        worst = bench.max_over_ranks(ms, "cpu")
        out[rank] = (worst, bench.job_tokens_per_s(world, 4096, 20, worst))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_throughput_two_ranks():
    world = 2
    port = _free_port()
    with mp.get_context("spawn").Manager() as m:
        out = m.dict()
        mp.spawn(_worker, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert res[0][0] == res[1][0] == 17.5
    assert abs(res[0][1] - 2 * 4096 * 20 / 0.0175) < 1e-6 * res[0][1]


def test_single_process_needs_no_collective():
    assert bench.max_over_ranks(3.25, "cpu") == 3.25
    assert bench.job_tokens_per_s(1, 64, 10, 5.0) == 64 * 10 / 0.005
