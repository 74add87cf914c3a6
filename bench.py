"""Benchmark of the cluster-routed sparse attention layer on B200.

Workload: the Wan-2.1-14B-class layer (B=1, H=40, L=75,600, d=128, bf16) with
ten simulated denoising steps: step 0 runs the full multi-stage clustering,
steps 1-9 warm-start from the previous step's centres (2 Lloyd iterations).
One bench "step" is that whole ten-step sequence over one layer: every row of
the hot path (query clustering, multi-stage / warm key clustering, stats and
permutations, Quest scores + top-k, sparse attention) runs inside the timed
region on inputs already resident in HBM (3 x 774 MB per denoising step, far
larger than L2).

metric: effective TFLOP/s = 10 x 4*B*H*L^2*d / t (dense-equivalent FLOPs of
the ten layer calls over their device time); higher is better.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Under torchrun every rank runs its own layer (independent problems, weak
scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

CONFIG_ID = 4
N_DENOISE = 10
NOISE_STD = 0.02


# ---------------------------------------------------------------- inputs
def max_over_ranks(ms_local, world, device, dist=None):
    """The job's time: the slowest rank's (every rank takes part, every rank gets it)."""
    import torch
    t = torch.tensor([ms_local], device=device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_tflops(ms, world, cfg):
    """Whole-job dense-equivalent rate: every rank runs one layer of cfg (weak scaling)."""
    return world * N_DENOISE * 4.0 * cfg.B * cfg.H * cfg.L * cfg.L * cfg.d / (ms * 1e-3) / 1e12


def _gen_head(args):
    cfg, head = args
    from cluster_routed_sparse_b200 import synth
    g = synth
    q = g._head_queries_f32(cfg, head)
    k = g._head_keys_f32(cfg, head)
    v = g._head_values_f32(cfg, head)
    return head, q, k, v


def generate_step0_f32(cfg, heads, procs: int):
    """fp32 step-0 tokens of the listed heads, generated in a spawn pool."""
    import multiprocessing as mp
    out = np.empty((3, len(heads), cfg.L, cfg.d), np.float32)
    ctx = mp.get_context("spawn")
    with ctx.Pool(procs) as pool:
        for h, q, k, v in pool.imap_unordered(_gen_head, [(cfg, h) for h in heads]):
            i = heads.index(h)
            out[0, i], out[1, i], out[2, i] = q, k, v
    return out


def denoise_inputs(x0_f32, steps: int, seed: int, device):
    """bf16 [steps][3][1,H,L,d] on the device: step 0 from the synthetic
    generator, step s = step s-1 + N(0, 0.02^2) (fp32 random walk, seeded
    CUDA generator), each rounded to bf16."""
    import torch
    x = torch.from_numpy(x0_f32).to(device)  # [3, H, L, d] fp32
    g = torch.Generator(device=device)
    out = []
    for s in range(steps):
        if s > 0:
            g.manual_seed(seed * 1000 + s)
            x += NOISE_STD * torch.randn(x.shape, generator=g, device=device, dtype=torch.float32)
        out.append([x[r].to(torch.bfloat16).unsqueeze(0).contiguous() for r in range(3)])
    del x
    return out


# ---------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during a region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": float(np.median(sm)) if sm else None, "sm_max_mhz": mx,
                "reasons": sorted(reasons), "samples": len(sm)}


# ---------------------------------------------------------------- CPU oracle leg
def oracle_sample(cfg_id: int, rows_attn: int = 256, heads=(0,)):
    """The oracle on a bounded sample of the workload: full step-0 clustering of
    the sampled heads (tau pooled over them), Quest + top-k, and attention for
    `rows_attn` query rows per head, extrapolated linearly to all L rows.
    Returns (effective TFLOP/s, extrapolated seconds of the sampled heads' layer,
    description, threads, wall seconds the sample itself took)."""
    from oracle import oracle as orc
    from cluster_routed_sparse_b200 import synth
    cfg = synth.CONFIGS[cfg_id]
    Q, K, V = synth.make_layer(cfg, heads=list(heads))
    Qf, Kf, Vf = (x.reshape(-1, cfg.L, cfg.d) for x in (Q, K, V))
    p = orc.Params.from_layer_config(cfg)
    t0 = time.perf_counter()
    r = orc.layer(Qf, Kf, Vf, p, attention=False)
    t1 = time.perf_counter()
    rows = np.linspace(0, cfg.L - 1, rows_attn).astype(np.int64)
    for h in range(len(heads)):
        orc.attention_rows(Qf[h], Kf[h], Vf[h], r.labels_q[h], r.kc.labels[h], r.sel[h], bool(r.kc.F[h]), rows)
    t2 = time.perf_counter()
    t_total = (t1 - t0) + (t2 - t1) * cfg.L / rows_attn
    t_wall = t2 - t0
    flops = 4.0 * len(heads) * cfg.L * cfg.L * cfg.d
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    desc = (f"{len(heads)} of {cfg.H} heads, step 0: full clustering + Quest/top-k; attention on "
            f"{rows_attn} of {cfg.L} query rows, extrapolated linearly")
    return flops / t_total / 1e12, t_total, desc, threads, t_wall


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    vals = []
    desc, threads = "", 1
    for i in range(args.warmup + args.steps):
        v, t, desc, threads, _ = oracle_sample(CONFIG_ID, rows_attn=128)
        if i >= args.warmup:
            vals.append((v, t))
    value = float(np.mean([v for v, _ in vals]))
    ms = float(np.mean([t for _, t in vals])) * 1e3
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic", "config": workload_config(),
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads, "kind": "oracle",
                            "sample": desc},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


METRIC = "sparse-attn layer ms & effective TFLOP/s (L=75,600 H=40 d=128) vs dense SDPA"


def workload_config():
    from cluster_routed_sparse_b200 import synth
    c = synth.CONFIGS[CONFIG_ID]
    return {"workload": f"{c.name}: B={c.B} H={c.H} L={c.L} d={c.d} bf16, {N_DENOISE} denoising steps "
                        f"(step 0 multi-stage, 9 warm), Cq={c.Cq}, m0={c.m0}, N_max={c.n_max}, "
                        f"tau=1.5x mean, top-k 10% of key clusters",
            "global_batch": c.B, "seq_len": c.L, "heads": c.H, "head_dim": c.d,
            "l2": "inputs larger than L2 (3 x 774 MB per denoising step, 10 distinct steps)",
            "parallelism": "one layer per rank"}


# ---------------------------------------------------------------- main
# DRAM bytes (read + write) of one k_sparse_attn launch per head, from the ncu capture summarised
# in profiles/k_sparse_attn_wan14b_h8.md (8 heads, scaled by heads), valid only for the kernel
# source it was taken on: any change to attn_kernel.cu turns the figure into null.
ATTN_TRAFFIC = {"sha256_prefix": "f0e4b1ad3dc6ebe4", "bytes_per_head": (313.705472e6 + 132.507648e6) / 8}


def attn_traffic_bytes(heads):
    import hashlib
    src = os.path.join(ROOT, "cluster_routed_sparse_b200", "csrc", "attn_kernel.cu")
    with open(src, "rb") as f:
        digest = hashlib.sha256(f.read()).hexdigest()
    if not digest.startswith(ATTN_TRAFFIC["sha256_prefix"]):
        return None
    return round(ATTN_TRAFFIC["bytes_per_head"] * heads)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sdpa", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--procs", type=int, default=min(32, os.cpu_count() or 1))
    ap.add_argument("--heads", type=int, default=0,
                    help="run only the first N heads (profiling of a smaller case; not a bench line)")
    args = ap.parse_args()
    if args.impl == "reference":
        return run_reference(args)

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    from cluster_routed_sparse_b200 import synth
    import dataclasses
    cfg = synth.CONFIGS[CONFIG_ID]
    if args.heads:
        cfg = dataclasses.replace(cfg, H=args.heads)

    # inputs first (spawn pool, before any CUDA call); each rank its own layer
    x0 = generate_step0_f32(cfg, list(range(cfg.H)), max(1, args.procs // max(1, world)))

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    from cluster_routed_sparse_b200.api import SparseLayer

    steps_in = denoise_inputs(x0, N_DENOISE, seed=100 + rank, device=dev)
    lay = SparseLayer.from_config(cfg, seed=1234 + rank)
    O = torch.empty_like(steps_in[0][0])

    def one_step(collect=None):
        for s in range(N_DENOISE):
            Q, K, V = steps_in[s]
            if collect is None:
                lay.forward(Q, K, V, O, warm=s > 0)
            else:
                _, t = lay.forward(Q, K, V, O, warm=s > 0, times=True)
                collect.append(t)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    launches0 = lay.launch_count()
    for _ in range(args.warmup):
        one_step()
    lay.synchronize()

    # ---- timed region
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    launches1 = lay.launch_count()
    e0.record(stream)
    per_call = []
    for _ in range(args.steps):
        one_step(per_call)
    e1.record(stream)
    barrier()
    clk = clocks.stop()
    launches = lay.launch_count() - launches1
    lay.synchronize()
    ms_local = e0.elapsed_time(e1) / args.steps
    ms = max_over_ranks(ms_local, world, dev, dist if world > 1 else None)

    dense_flops_layer = 4.0 * cfg.B * cfg.H * cfg.L * cfg.L * cfg.d
    value = job_tflops(ms, world, cfg)

    # stage split (from the same timed calls)
    step0 = [c for i, c in enumerate(per_call) if i % N_DENOISE == 0]
    warm = [c for i, c in enumerate(per_call) if i % N_DENOISE != 0]
    avg = lambda rows, k: float(np.mean([r[k] for r in rows]))  # noqa: E731
    keys = ["q_cluster_ms", "k_cluster_ms", "stats_sort_ms", "score_select_ms", "attention_ms",
            "attn_kernel_ms", "total_ms"]
    split0 = {k: avg(step0, k) for k in keys}
    splitw = {k: avg(warm, k) for k in keys}
    cnt = lay.counters()

    # roofline of the dominant kernel (sparse attention, tensor-bound)
    peaks = {}
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            peaks = json.load(f)
    except Exception:
        pass
    peak_tf = peaks.get("bf16_tflops_sustained")
    peak_src = "of measured (bf16_tflops_sustained)" if peak_tf else "of fallback"
    peak_tf = peak_tf or 1400.0
    attn_flops = 4.0 * cfg.d * cnt["kept_pairs"]  # last call (a warm step)
    traffic = attn_traffic_bytes(cfg.H)
    achieved = attn_flops / (splitw["attn_kernel_ms"] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_tf, "unit": "TFLOP/s",
                "frac": round(achieved / peak_tf, 4), "traffic": traffic, "peak_source": peak_src,
                "kernel": "k_sparse_attn (warm-step launch)",
                "algorithmic_flops_per_launch": attn_flops,
                "computed_tile_flops_per_launch": 4.0 * cfg.d * cnt["computed_pairs"],
                "computed_frac": round(4.0 * cfg.d * cnt["computed_pairs"] / (splitw["attn_kernel_ms"] * 1e-3) / 1e12
                                       / peak_tf, 4)}
    # achieved HBM fraction of the reduction stages of a warm call: the bytes they must read
    # (a tensor of B*H*L*d bf16 per pass) over their measured time
    hbm = peaks.get("hbm_gbs") or 6650.0
    tensor_bytes = 2.0 * cfg.B * cfg.H * cfg.L * cfg.d
    passes = {"q_cluster_ms": 1 + 3 + 2,   # norms, 3 assignment passes, 2 centre updates
              "k_cluster_ms": 1 + 3 + 2,   # norms, 3 passes, 2 updates
              "stats_sort_ms": 1}          # per-cluster max / min, exact distances, SSE (one pass)
    red = {}
    for k, n in passes.items():
        gbs = n * tensor_bytes / (splitw[k] * 1e-3) / 1e9
        red[k.replace("_ms", "")] = {"algorithmic_bytes": n * tensor_bytes, "ms": round(splitw[k], 3),
                                     "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / hbm, 4)}

    extra = {"step0": split0, "warm": splitw, "counters_last_call": cnt,
             "reduction_stages_hbm": red,
             "clustering_share_warm": round((splitw["q_cluster_ms"] + splitw["k_cluster_ms"] + splitw["stats_sort_ms"]
                                             + splitw["score_select_ms"]) / splitw["total_ms"], 4),
             "assign_counters_since_create": lay.assign_counters(),
             "kept_pair_frac": cnt["kept_pairs"] / float(cfg.H * cfg.L * cfg.L),
             "tile_efficiency": cnt["kept_pairs"] / max(1, cnt["computed_pairs"])}
    # per-head state after the last call: key clusters, dense fallback, compactness, step-0 stages
    try:
        from cluster_routed_sparse_b200 import _lib as L
        extra["per_head"] = {
            "n_k": lay.tensor(L.AC_T_N_K).cpu().tolist(),
            "dense": lay.tensor(L.AC_T_DENSE).cpu().tolist(),
            "comp": [round(float(x), 5) for x in lay.tensor(L.AC_T_COMP).cpu().tolist()],
            "stages": lay.tensor(L.AC_T_STAGES).cpu().tolist()}
    except Exception as exc:  # reporting only: never fail the bench line on it
        extra["per_head"] = {"unavailable": str(exc)[:200]}
    # dense SDPA on the same tensors (one warm step's inputs)
    if not args.no_sdpa and rank == 0:
        extra["dense_sdpa"] = time_sdpa(*steps_in[1])
        if extra["dense_sdpa"].get("ms"):
            sd = extra["dense_sdpa"]["ms"]
            extra["speedup_warm_layer_vs_sdpa"] = sd / splitw["total_ms"]
            extra["speedup_sequence_vs_sdpa"] = sd * N_DENOISE / ms

    # e2e through the host-buffer entry point
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(lay, steps_in, cfg, dense_flops_layer, world, dist if world > 1 else None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, tsec, desc, threads, twall = oracle_sample(CONFIG_ID)
        cpu = {"value": v, "unit": "TFLOP/s", "cores": threads, "kind": "oracle", "sample": desc,
               "extrapolated_seconds": tsec, "sample_wall_seconds": twall}

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
               "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(),
               "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
               "clocks": clk, "layer_ms_warm": splitw["total_ms"], "layer_ms_step0": split0["total_ms"],
               "extra": extra}
        print(json.dumps(out), flush=True)
    lay.close()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def time_sdpa(Q, K, V, reps: int = 3):
    import torch
    from torch.nn.attention import SDPBackend, sdpa_kernel
    F = torch.nn.functional
    for be, name in ((SDPBackend.CUDNN_ATTENTION, "cudnn"), (SDPBackend.FLASH_ATTENTION, "flash"),
                     (SDPBackend.EFFICIENT_ATTENTION, "efficient")):
        try:
            with sdpa_kernel([be]):
                F.scaled_dot_product_attention(Q, K, V)
                torch.cuda.synchronize()
                ts = []
                for _ in range(reps):
                    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    a.record()
                    F.scaled_dot_product_attention(Q, K, V)
                    b.record()
                    torch.cuda.synchronize()
                    ts.append(a.elapsed_time(b))
            ms = float(np.median(ts))
            fl = 4.0 * Q.shape[0] * Q.shape[1] * Q.shape[2] * K.shape[2] * Q.shape[3]
            return {"backend": name, "ms": ms, "tflops": fl / (ms * 1e-3) / 1e12}
        except Exception as e:  # backend unavailable for this shape
            last = str(e)[:200]
    return {"backend": None, "ms": None, "error": last}


def time_e2e(lay, steps_in, cfg, dense_flops_layer, world, dist):
    """One ten-step sequence through the asynchronous host-buffer entry point
    (ac_layer_forward_host_async): every call copies that step's Q, K, V from
    pinned host memory and O back; a call's copies overlap its neighbours'
    layers.  Timed from before the first call's input copy to the end of the
    last call's output copy (ac_join on the timing stream)."""
    import torch
    host = []
    for s in range(N_DENOISE):
        host.append([x.cpu().pin_memory() for x in steps_in[s]])
    hO = torch.empty_like(host[0][0]).pin_memory()
    torch.cuda.synchronize()
    lay.forward_host_async(*host[0], hO, warm=False)  # warm-up of the staging buffers and streams
    lay.synchronize()
    stream = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for s in range(N_DENOISE):
        lay.forward_host_async(*host[s], hO, warm=s > 0)
    lay.join()
    e1.record(stream)
    torch.cuda.synchronize()
    lay.synchronize()
    ms = e0.elapsed_time(e1)
    if dist is not None:
        t = torch.tensor([ms], device="cuda", dtype=torch.float64)
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        ms = float(t.item())
    nbytes = cfg.B * cfg.H * cfg.L * cfg.d * 2
    return {"value": world * N_DENOISE * dense_flops_layer / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": 3 * nbytes * N_DENOISE, "d2h_bytes_per_step": nbytes * N_DENOISE,
            "ms_per_step": ms, "api": "ac_layer_forward_host_async x 10, ac_join",
            "clock": "CUDA events around the ten host-buffer calls"}


if __name__ == "__main__":
    sys.exit(main())
