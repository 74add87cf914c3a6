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


def test_attention_traffic_is_tied_to_the_captured_sources(tmp_path, monkeypatch):
    """roofline.traffic is an ncu figure of one kernel version: it is reported
    for the bench workload only while the hashed kernel sources are the ones
    it was captured on, and turns null once either file changes."""
    sys.path.insert(0, ROOT)
    import shutil
    import bench
    from cluster_routed_sparse_b200 import synth
    cfg = synth.CONFIGS[bench.CONFIG_ID]
    assert cfg.name == "wan14b-L75600-H40-d128"
    assert bench.attn_traffic_bytes(cfg) == round(bench.ATTN_TRAFFIC["bytes_per_head"] * cfg.H)
    assert all(bench.attn_traffic_bytes(c) is None for c in synth.CONFIGS.values() if c.name != cfg.name)
    csrc = tmp_path / "cluster_routed_sparse_b200" / "csrc"
    csrc.mkdir(parents=True)
    for name in ("attn_kernel.cu", "ac_device.cuh"):
        shutil.copy(os.path.join(ROOT, "cluster_routed_sparse_b200", "csrc", name), csrc / name)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.attn_traffic_bytes(cfg) is not None
    with open(csrc / "ac_device.cuh", "a") as f:
        f.write("\n// edited\n")
    assert bench.attn_traffic_bytes(cfg) is None
