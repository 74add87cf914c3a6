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


def test_reference_arm_prints_one_contract_line_on_the_small_workload():
    """`bench.py --impl reference` times the oracle on the host cores and prints
    one JSON line with the arm's keys (run here on the small workload)."""
    import json
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--config", "1",
                          "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s" and d["higher_is_better"] is True
    assert d["steps"] == 2 and d["warmup"] == 1 and d["n_gpus"] == 1
    assert d["value"] > 0 and d["ms_per_step"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
