"""The multi-GPU bench arithmetic on CPU: two gloo ranks (one process each,
127.0.0.1), each with its own step time; every rank must get the slowest
rank's time, and the whole-job rate must count both ranks' layers."""
import os
import socket
import sys

import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    import bench
    from cluster_routed_sparse_b200 import synth
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        ms = bench.max_over_ranks(100.0 + 7.0 * rank, world, "cpu", dist)
        cfg = synth.CONFIGS[bench.CONFIG_ID]
        out[rank] = (ms, bench.job_tflops(ms, world, cfg), bench.job_tflops(ms, 1, cfg))
    finally:
        dist.destroy_process_group()


def test_two_rank_max_and_weak_scaling_rate():
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    assert sorted(res) == [0, 1]
    for r in range(world):
        ms, v2, v1 = res[r]
        assert ms == 107.0
        assert abs(v2 - 2 * v1) < 1e-9 * v1
    # the rate at 107 ms for one layer of the bench workload, by hand
    L, H, d = 75600, 40, 128
    expect = 2 * 10 * 4.0 * H * L * L * d / 0.107 / 1e12
    assert abs(res[0][1] - expect) < 1e-6 * expect


def test_single_rank_needs_no_process_group():
    sys.path.insert(0, ROOT)
    import bench
    assert bench.max_over_ranks(12.5, 1, "cpu") == 12.5
