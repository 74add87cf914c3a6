"""Benchmark of the cluster-routed sparse attention layer on B200.

Default workload: the Wan-2.1-14B-class layer (B=1, H=40, L=75,600, d=128,
bf16) with ten simulated denoising steps: step 0 runs the full multi-stage
clustering, steps 1-9 warm-start from the previous step's centres (2 Lloyd
iterations).  One bench "step" is that whole ten-step sequence over one layer:
every row of the hot path (query clustering, multi-stage / warm key
clustering, stats and permutations, Quest scores + top-k, sparse attention)
runs inside the timed region on inputs already resident in HBM (3 x 774 MB per
denoising step, far larger than L2).  --config N selects another workload of
synth.CONFIGS (one step-0 layer call per bench step; L2 flushed between bench
steps, outside the timed events).

metric: effective TFLOP/s = calls x 4*B*H*L^2*d / t (dense-equivalent FLOPs of
the layer calls over their device time); higher is better.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--config N] [--topk -PERMILLE] [--stage-rule R] [--tail-merge M] [--compensate]

Under torchrun every rank runs its own layer (independent problems, weak
scaling, no collective on the data path); time is the max over ranks.
"""
from __future__ import annotations

import argparse
import json
import os
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

DEFAULT_CONFIG = 4
CONFIG_ID = DEFAULT_CONFIG
NOISE_STD = 0.02
METRIC = "sparse-attn layer ms & effective TFLOP/s (L=75,600 H=40 d=128) vs dense SDPA"


def workload(args):
    """The synth.LayerConfig the run measures (with any overrides)."""
    import dataclasses
    from cluster_routed_sparse_b200 import synth
    cfg = synth.CONFIGS[args.config]
    over = {}
    if args.topk:
        over["topk"] = args.topk
    if args.stage_rule is not None:
        over["stage_rule"] = args.stage_rule
    if args.heads:
        over["H"] = args.heads
    return dataclasses.replace(cfg, **over) if over else cfg


def tau_text(cfg):
    return {0: f"tau={cfg.tau_value:g}", 1: f"tau={cfg.tau_value:g}x mean",
            2: f"tau=p{cfg.tau_value / 10:g} of the stage-0 distances"}[cfg.tau_mode]


def workload_config(cfg, args):
    steps = cfg.steps
    seq = (f"{steps} denoising steps (step 0 multi-stage, {steps - 1} warm)" if steps > 1
           else "one step-0 layer call (multi-stage key clustering)")
    topk = f"top-k {-cfg.topk / 10:g}% of key clusters" if cfg.topk < 0 else f"top-k {cfg.topk}"
    return {"workload": f"{cfg.name}: B={cfg.B} H={cfg.H} L={cfg.L} d={cfg.d} bf16, {seq}, Cq={cfg.Cq}, "
                        f"m0={cfg.m0}, N_max={cfg.n_max}, {tau_text(cfg)}, {topk}, stage rule {cfg.stage_rule}"
                        + (f", tail merging {args.tail_merge}" if args.tail_merge else "")
                        + (", centroid compensation" if args.compensate else ""),
            "global_batch": cfg.B, "seq_len": cfg.L, "heads": cfg.H, "head_dim": cfg.d,
            "l2": ("inputs larger than L2 (3 x 774 MB per denoising step, 10 distinct steps)" if steps > 1
                   else "L2 flushed (512 MB write) before every timed bench step, outside its events"),
            "parallelism": ("the layer's heads split over the ranks, tau pooled by an NCCL all-reduce"
                            if getattr(args, "split_heads", False) else "one layer per rank")}


# ---------------------------------------------------------------- inputs
def max_over_ranks(ms_local, world, device, dist=None):
    """The job's time: the slowest rank's (every rank takes part, every rank gets it)."""
    import torch
    t = torch.tensor([ms_local], device=device, dtype=torch.float64)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def dense_flops(cfg):
    return 4.0 * cfg.B * cfg.H * cfg.L * cfg.L * cfg.d


def job_tflops(ms, world, cfg):
    """Whole-job dense-equivalent rate: every rank runs one layer of cfg, cfg.steps
    calls per bench step (weak scaling)."""
    return world * cfg.steps * dense_flops(cfg) / (ms * 1e-3) / 1e12


def _gen_head(args):
    cfg, head = args
    from cluster_routed_sparse_b200 import synth
    return head, synth._head_queries_f32(cfg, head), synth._head_keys_f32(cfg, head), synth._head_values_f32(cfg, head)


def generate_step0_f32(cfg, heads, procs: int):
    """fp32 step-0 tokens of the listed heads, generated in a spawn pool."""
    import multiprocessing as mp
    out = np.empty((3, len(heads), cfg.L, cfg.d), np.float32)
    with mp.get_context("spawn").Pool(procs) as pool:
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


# ---------------------------------------------------------------- CPU oracle legs
class OracleSample:
    """The oracle, as it stands, on a bounded sample of one head of the workload:
    step-0 clustering (tau from that head's own distances), Quest + top-k and
    attention for `rows` query rows; with warm steps in the workload, also one
    warm-started step of the same head.  Attention is extrapolated linearly to
    all L rows; the head's sequence time is t0 + (steps - 1) * t_warm."""

    def __init__(self, cfg, rows: int = 128, head: int = 0):
        from oracle import oracle as orc
        from cluster_routed_sparse_b200 import synth
        self.orc, self.cfg, self.rows = orc, cfg, rows
        Q, K, V = synth.make_layer(cfg, heads=[head])
        self.Q, self.K, self.V = (x.reshape(-1, cfg.L, cfg.d) for x in (Q, K, V))
        self.p = orc.Params.from_layer_config(cfg)
        self.rowsel = np.linspace(0, cfg.L - 1, rows).astype(np.int64)
        self.r0 = None
        self.t0 = self.tw = None

    def _attn(self, r):
        self.orc.attention_rows(self.Q[0], self.K[0], self.V[0], r.labels_q[0], r.kc.labels[0], r.sel[0],
                                bool(r.kc.F[0]), self.rowsel)

    def step0(self):
        a = time.perf_counter()
        self.r0 = self.orc.layer(self.Q, self.K, self.V, self.p, attention=False)
        b = time.perf_counter()
        self._attn(self.r0)
        c = time.perf_counter()
        self.t0 = (b - a) + (c - b) * self.cfg.L / self.rows
        return c - a

    def warm(self):
        if self.r0 is None:
            self.step0()
        a = time.perf_counter()
        r = self.orc.layer(self.Q, self.K, self.V, self.p, warm_from=self.r0, attention=False)
        b = time.perf_counter()
        self._attn(r)
        c = time.perf_counter()
        self.tw = (b - a) + (c - b) * self.cfg.L / self.rows
        return c - a

    def sequence_seconds(self):
        steps = self.cfg.steps
        return self.t0 + (steps - 1) * (self.tw if steps > 1 else 0.0)

    def tflops(self):
        return self.cfg.steps * 4.0 * self.cfg.L * self.cfg.L * self.cfg.d / self.sequence_seconds() / 1e12

    def describe(self):
        w = (f" + one warm step ({self.cfg.iters_warm} Lloyd iterations), sequence time t0 + "
             f"{self.cfg.steps - 1} x t_warm" if self.cfg.steps > 1 else "")
        return (f"1 of {self.cfg.H} heads: step-0 clustering (tau from that head's distances) + Quest/top-k"
                f"{w}; attention on {self.rows} of {self.cfg.L} query rows per step, extrapolated linearly")


def threads_used():
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))


def run_reference(args):
    """The reference arm: the oracle timed on the host cores (rank 0 only)."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    cfg = workload(args)
    smp = OracleSample(cfg, rows=128)
    # each step: the step-0 sample, or (workloads with warm steps) alternately the
    # step-0 and the warm-step sample; warm-up steps run the attention rows only
    for _ in range(args.warmup):
        if smp.r0 is None:
            smp.step0()
        else:
            smp._attn(smp.r0)
    walls = []
    for i in range(args.steps):
        walls.append(smp.warm() if (cfg.steps > 1 and i % 2 == 1) else smp.step0())
    if cfg.steps > 1 and smp.tw is None:
        smp.warm()
    value = smp.tflops()
    ms = float(np.mean(walls)) * 1e3
    out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "impl": "reference",
           "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
           "ms_per_step_note": "wall time of each step's oracle sample (one head); value is that head's "
                               "extrapolated sequence rate",
           "extrapolated_head_sequence_ms": smp.sequence_seconds() * 1e3,
           "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
           "data": "synthetic", "config": workload_config(cfg, args),
           "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": threads_used(), "kind": "oracle",
                            "sample": smp.describe()},
           "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)
    return 0


# ---------------------------------------------------------------- main
# DRAM bytes (read + write) of one k_sparse_attn launch per head of the bench
# workload, from an ncu capture of its 8-head reduction, valid only for the
# kernel source it was taken on: any change to attn_kernel.cu or to the device
# helpers it includes (ac_device.cuh) turns it into null.
ATTN_TRAFFIC = {"sha256_prefix": "59005465043a9f46", "bytes_per_head": (313656320 + 128224768) / 8}


def attn_source_digest():
    import hashlib
    h = hashlib.sha256()
    for name in ("attn_kernel.cu", "ac_device.cuh"):
        with open(os.path.join(ROOT, "cluster_routed_sparse_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


def attn_traffic_bytes(cfg):
    if cfg.name != "wan14b-L75600-H40-d128":
        return None
    if not attn_source_digest().startswith(ATTN_TRAFFIC["sha256_prefix"]):
        return None
    return round(ATTN_TRAFFIC["bytes_per_head"] * cfg.H)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--config", type=int, default=DEFAULT_CONFIG, help="workload id in synth.CONFIGS")
    ap.add_argument("--topk", type=int, default=0, help="override the top-k (negative: -permille of n_k)")
    ap.add_argument("--stage-rule", type=int, default=None, help="override the m_t rule of stages t > 0")
    ap.add_argument("--tail-merge", type=int, default=0, help="query-tile tail merging mode (0, 1, 2)")
    ap.add_argument("--compensate", action="store_true",
                    help="centroid compensation of the unselected key clusters")
    ap.add_argument("--e2e-reps", type=int, default=3, help="repetitions of the end-to-end measurement")
    ap.add_argument("--split-heads", action="store_true",
                    help="under torchrun: one layer, its heads split over the ranks (strong scaling), the "
                         "step-0 tau pooled by an all-reduce")
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
    cfg = workload(args)
    n_calls = cfg.steps  # layer calls per bench step

    # inputs first (spawn pool, before any CUDA call); each rank its own layer
    split = args.split_heads and world > 1
    h_lo, h_hi = (rank * cfg.H // world, (rank + 1) * cfg.H // world) if split else (0, cfg.H)
    heads = list(range(h_lo, h_hi))
    import dataclasses
    lcfg = dataclasses.replace(cfg, H=len(heads)) if split else cfg  # this rank's share
    x0 = generate_step0_f32(cfg, heads, max(1, args.procs // max(1, world)))

    import torch
    import torch.distributed as dist
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=300), device_id=dev)
    from cluster_routed_sparse_b200.api import SparseLayer

    steps_in = denoise_inputs(x0, n_calls, seed=100 + (h_lo if split else rank), device=dev)
    del x0
    if split:
        # this rank's heads of the one layer; the initial centres keep each head's
        # seeds and the step-0 tau is pooled over all ranks (ac_set_tau_exchange)
        from cluster_routed_sparse_b200.api import tau_exchange_allreduce
        lay = SparseLayer.from_config(cfg, seed=1234, H=len(heads), tail_merge=args.tail_merge,
                                      compensate=1 if args.compensate else 0, unit0=h_lo)
        lay.set_tau_exchange(tau_exchange_allreduce(device=dev))
    else:
        lay = SparseLayer.from_config(cfg, seed=1234 + rank, tail_merge=args.tail_merge,
                                      compensate=1 if args.compensate else 0)
    O = torch.empty_like(steps_in[0][0])
    flush_buf = torch.empty(512 << 20, dtype=torch.uint8, device=dev)

    def one_step(collect=None):
        for s in range(n_calls):
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

    for _ in range(args.warmup):
        one_step()
    lay.synchronize()

    # ---- timed region: K bench steps, each between its own events on the
    # launching stream; the L2 flush before each step lies outside them
    stream = torch.cuda.current_stream()
    clocks = ClockSampler(local)
    barrier()
    clocks.start()
    launches1 = lay.launch_count()
    per_call, ev = [], []
    for _ in range(args.steps):
        flush_buf.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        one_step(per_call)
        e1.record(stream)
        ev.append((e0, e1))
    barrier()
    clk = clocks.stop()
    launches = lay.launch_count() - launches1
    lay.synchronize()
    ms_local = sum(a.elapsed_time(b) for a, b in ev) / args.steps
    ms = max_over_ranks(ms_local, world, dev, dist if world > 1 else None)
    value = job_tflops(ms, 1 if split else world, cfg)

    # stage split (from the same timed calls): step 0 and the warm steps
    step0 = [c for i, c in enumerate(per_call) if i % n_calls == 0]
    warm = [c for i, c in enumerate(per_call) if i % n_calls != 0]
    keys = ["q_cluster_ms", "k_cluster_ms", "stats_sort_ms", "score_select_ms", "attention_ms",
            "attn_kernel_ms", "total_ms"]
    avg = lambda rows, k: float(np.mean([r[k] for r in rows]))  # noqa: E731
    split0 = {k: avg(step0, k) for k in keys}
    splitw = {k: avg(warm, k) for k in keys} if warm else None
    steady = splitw or split0  # the call the roofline and the SDPA comparison use
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
    attn_flops = 4.0 * cfg.d * cnt["kept_pairs"]  # last call (a warm step when there are warm steps)
    achieved = attn_flops / (steady["attn_kernel_ms"] * 1e-3) / 1e12
    roofline = {"bound": "tensor", "achieved": round(achieved, 2), "peak": peak_tf, "unit": "TFLOP/s",
                "frac": round(achieved / peak_tf, 4), "traffic": attn_traffic_bytes(lcfg), "peak_source": peak_src,
                "kernel": "k_sparse_attn (" + ("warm-step launch" if warm else "step-0 launch") + ")",
                "algorithmic_flops_per_launch": attn_flops,
                "computed_tile_flops_per_launch": 4.0 * cfg.d * cnt["computed_pairs"],
                "computed_frac": round(4.0 * cfg.d * cnt["computed_pairs"] / (steady["attn_kernel_ms"] * 1e-3)
                                       / 1e12 / peak_tf, 4)}
    # achieved HBM fraction of the reduction stages: the bytes they must read
    # (a tensor of B*H*L*d bf16 per pass) over their measured time
    hbm = peaks.get("hbm_gbs") or 6650.0
    tensor_bytes = 2.0 * lcfg.B * lcfg.H * lcfg.L * lcfg.d
    passes = ({"q_cluster_ms": 1 + (cfg.iters_warm + 1) + cfg.iters_warm,   # norms, assignment passes, updates
               "k_cluster_ms": 1 + (cfg.iters_warm + 1) + cfg.iters_warm,
               "stats_sort_ms": 1} if warm else
              {"q_cluster_ms": 1 + (cfg.iters_q + 1) + cfg.iters_q, "stats_sort_ms": 1})
    red = {}
    for k, n in passes.items():
        gbs = n * tensor_bytes / (steady[k] * 1e-3) / 1e9
        red[k.replace("_ms", "")] = {"algorithmic_bytes": n * tensor_bytes, "ms": round(steady[k], 3),
                                     "GB/s": round(gbs, 1), "frac_of_measured_hbm": round(gbs / hbm, 4)}

    clustering_ms = steady["total_ms"] - steady["attention_ms"]
    extra = {"step0": split0, "warm": splitw, "counters_last_call": cnt,
             "reduction_stages_hbm": red,
             "clustering_share": round(clustering_ms / steady["total_ms"], 4),
             "assign_counters_since_create": lay.assign_counters(),
             "kept_pair_frac": cnt["kept_pairs"] / float(lcfg.B * lcfg.H * lcfg.L * lcfg.L),
             "tile_efficiency": cnt["kept_pairs"] / max(1, cnt["computed_pairs"])}
    try:
        from cluster_routed_sparse_b200 import _lib as L
        n_k = lay.tensor(L.AC_T_N_K).cpu().numpy()
        ksel = lay.tensor(L.AC_T_KSEL).cpu().numpy()
        dense = lay.tensor(L.AC_T_DENSE).cpu().numpy()
        sparse = dense == 0
        extra["kept_cluster_frac"] = float(np.mean(ksel[sparse] / n_k[sparse])) if sparse.any() else 1.0
        extra["per_head"] = {"n_k": n_k.tolist(), "dense": dense.tolist(),
                             "comp": [round(float(x), 5) for x in lay.tensor(L.AC_T_COMP).cpu().tolist()],
                             "stages": lay.tensor(L.AC_T_STAGES).cpu().tolist()}
    except Exception as exc:  # reporting only: never fail the bench line on it
        extra["per_head"] = {"unavailable": str(exc)[:200]}
    # dense SDPA on the same tensors (a warm step's inputs when there are warm steps)
    if not args.no_sdpa and rank == 0:
        sd = time_sdpa(*steps_in[1 if n_calls > 1 else 0])
        extra["dense_sdpa"] = sd
        if sd.get("ms"):
            extra["speedup_layer_vs_sdpa"] = sd["ms"] / steady["total_ms"]
            extra["speedup_sequence_vs_sdpa"] = sd["ms"] * n_calls / ms
            # What the kept pairs allow: the layer cannot beat SDPA by more than
            # t_sdpa / (t_clustering + kept FLOPs at the peak rate), nor, with free
            # clustering, by more than t_sdpa / (kept FLOPs at the peak rate).
            t_attn_peak = attn_flops / (peak_tf * 1e12) * 1e3
            extra["speedup_bound_at_peak"] = sd["ms"] / (clustering_ms + t_attn_peak)
            extra["speedup_bound_free_clustering"] = sd["ms"] / t_attn_peak
            extra["speedup_bound_note"] = ("t_sdpa / (measured clustering + selection ms + kept-pair FLOPs at "
                                           f"{peak_tf} TFLOP/s); the second bound drops the clustering")

    # e2e through the asynchronous host-buffer entry point
    e2e = None
    if not args.no_e2e:
        e2e = time_e2e(lay, steps_in, lcfg, args, 1 if split else world, dist if world > 1 else None,
                       job_flops=cfg.steps * dense_flops(cfg) if split else None)

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        smp = OracleSample(cfg, rows=256)
        wall = smp.step0() + (smp.warm() if cfg.steps > 1 else 0.0)
        cpu = {"value": smp.tflops(), "unit": "TFLOP/s", "cores": threads_used(), "kind": "oracle",
               "sample": smp.describe(), "extrapolated_head_sequence_seconds": smp.sequence_seconds(),
               "sample_wall_seconds": wall}

    if rank == 0:
        out = {"metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world, "steps": args.steps,
               "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
               "scaling": "strong" if split else "weak",
               "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": workload_config(cfg, args),
               "roofline": roofline, "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches,
               "clocks": clk, "layer_ms_step0": split0["total_ms"],
               "layer_ms_warm": splitw["total_ms"] if splitw else None, "extra": extra}
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
    last = None
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


def time_e2e(lay, steps_in, cfg, args, world, dist, job_flops=None):
    """The bench steps through the asynchronous host-buffer entry point
    (ac_layer_forward_host_async): every call copies that step's Q, K, V from
    pinned host memory and O back; a call's copies overlap its neighbours'
    layers.  Each repetition times args.steps bench steps back to back, from
    before the first call's input copy to the end of the last call's output copy
    (ac_join on the timing stream); the value is the median repetition."""
    import torch
    n_calls = cfg.steps
    host = [[x.cpu().pin_memory() for x in steps_in[s]] for s in range(n_calls)]
    hO = torch.empty_like(host[0][0]).pin_memory()
    torch.cuda.synchronize()
    lay.forward_host_async(*host[0], hO, warm=False)  # warm-up of the staging buffers and streams
    lay.synchronize()
    stream = torch.cuda.current_stream()
    reps = []
    for _ in range(max(1, args.e2e_reps)):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        for _ in range(args.steps):
            for s in range(n_calls):
                lay.forward_host_async(*host[s], hO, warm=s > 0)
        lay.join()
        e1.record(stream)
        torch.cuda.synchronize()
        lay.synchronize()
        ms = e0.elapsed_time(e1) / args.steps
        if dist is not None:
            t = torch.tensor([ms], device="cuda", dtype=torch.float64)
            dist.all_reduce(t, op=dist.ReduceOp.MAX)
            ms = float(t.item())
        reps.append(ms)
    ms = float(np.median(reps))
    nbytes = cfg.B * cfg.H * cfg.L * cfg.d * 2
    flops = job_flops if job_flops is not None else world * n_calls * dense_flops(cfg)
    return {"value": flops / (ms * 1e-3) / 1e12, "unit": "TFLOP/s",
            "h2d_bytes_per_step": 3 * nbytes * n_calls, "d2h_bytes_per_step": nbytes * n_calls,
            "ms_per_step": ms, "ms_per_step_reps": [round(x, 2) for x in reps],
            "api": f"ac_layer_forward_host_async x {n_calls} per step, ac_join",
            "clock": "CUDA events around each repetition's host-buffer calls"}


if __name__ == "__main__":
    sys.exit(main())
