"""Seeded synthetic Q/K/V for one video-DiT attention layer.

This module only draws random numbers and rounds them to bf16; it holds none of
the clustering, scoring or attention arithmetic.  Both the CUDA path (tests,
bench) and the CPU oracle take their inputs from here.

Recipe (stand-in for real DiT activations, which are not available):

* K: a mixture of Gaussian components per head.  Component centres are
  N(0, I_d); each component has its own per-dimension std drawn U(0.05, 0.3)
  (anisotropic).  Tokens pick a component (equal weights, or Dirichlet weights
  for the heavy-tailed workload) and are centre + std * N(0, I_d).  A "diffuse"
  head draws keys i.i.d. N(0, I_d) instead.
* Q: 16 unit directions per head; a token picks one, adds angular noise of
  size 0.2 and is rescaled by a lognormal(0, 0.7) norm.
* V: N(0, I_d).
* Denoising steps: step s adds N(0, 0.02^2) noise to the previous step's
  tokens (fp32), then rounds to bf16.

Every head has its own random stream, so any subset of heads can be
regenerated bit-identically.  Values are drawn in fp32 and rounded to bf16
with round-to-nearest-even.
"""
from __future__ import annotations

import dataclasses
import numpy as np

__all__ = [
    "LayerConfig", "CONFIGS", "f32_to_bf16_bits", "bf16_bits_to_f32",
    "make_layer", "make_head",
]


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape and method hyper-parameters of one synthetic layer workload."""
    name: str
    B: int
    H: int
    L: int
    d: int
    Cq: int                  # query clusters (angular k-means)
    m0: int                  # initial key clusters of the multi-stage k-means
    n_max: int               # cluster cap that triggers the dense fallback
    tau_mode: int            # 0 absolute, 1 factor x mean, 2 percentile (permille)
    tau_value: float         # tau, factor, or permille
    topk: int                # >0: clusters per query cluster; <0: -permille of n_k
    iters_q: int = 10
    iters_k: int = 10
    iters_warm: int = 2
    key_components: object = 48      # int, or (lo, hi) drawn per head
    dirichlet_alpha: float = 0.0     # >0: component weights ~ Dirichlet(alpha)
    diffuse_heads: tuple = ()
    q_directions: int = 16
    steps: int = 1                   # simulated denoising steps
    seed: int = 20260000
    stage_rule: int = 0              # m_t of stages t > 0: 0 = min(m0, |U|), 1 = proportional


TAU_ABSOLUTE, TAU_MEAN_FACTOR, TAU_PERCENTILE = 0, 1, 2

CONFIGS = {
    # Tiny CPU-checkable layer.
    1: LayerConfig("tiny-L4096-H2-d64", 1, 2, 4096, 64, Cq=16, m0=32, n_max=128,
                   tau_mode=TAU_MEAN_FACTOR, tau_value=0.5, topk=8,
                   key_components=48),
    # CogVideoX-2B-class layer; heads 0 and 1 diffuse -> dense fallback.
    2: LayerConfig("cogvideox2b-L17550-H30-d64", 1, 30, 17550, 64, Cq=65, m0=200,
                   n_max=600, tau_mode=TAU_MEAN_FACTOR, tau_value=1.5, topk=-100,
                   key_components=200, diffuse_heads=(0, 1)),
    # Wan-2.1-1.3B-class layer; per-head component count U(100, 600).
    3: LayerConfig("wan1.3b-L32760-H12-d128", 1, 12, 32760, 128, Cq=65, m0=256,
                   n_max=1000, tau_mode=TAU_PERCENTILE, tau_value=900.0,
                   topk=-100, key_components=(100, 600)),
    # Wan-2.1-14B-class layer at L=75,600 with warm-started denoising steps.
    4: LayerConfig("wan14b-L75600-H40-d128", 1, 40, 75600, 128, Cq=65, m0=256,
                   n_max=1000, tau_mode=TAU_MEAN_FACTOR, tau_value=1.5,
                   topk=-100, key_components=500, steps=10),
    # Long-sequence stress case with heavy-tailed cluster sizes.
    5: LayerConfig("long-L118800-H24-d128", 1, 24, 118800, 128, Cq=65, m0=256,
                   n_max=1500, tau_mode=TAU_MEAN_FACTOR, tau_value=1.5,
                   topk=-50, key_components=800, dirichlet_alpha=0.3),
}


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round fp32 to bf16 (round-to-nearest-even); returns uint16 bit patterns."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to fp32."""
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def _rng(cfg: LayerConfig, head: int, role: int, step: int = 0) -> np.random.Generator:
    return np.random.default_rng([cfg.seed + cfg.L, cfg.H, head, role, step])


def _head_keys_f32(cfg: LayerConfig, head: int) -> np.ndarray:
    L, d = cfg.L, cfg.d
    g = _rng(cfg, head, 1)
    if head in cfg.diffuse_heads:
        return g.standard_normal((L, d), dtype=np.float32)
    nc = cfg.key_components
    if isinstance(nc, tuple):
        nc = int(g.integers(nc[0], nc[1] + 1))
    mu = g.standard_normal((nc, d), dtype=np.float32)
    sd = g.uniform(0.05, 0.3, size=(nc, d)).astype(np.float32)
    if cfg.dirichlet_alpha > 0:
        w = g.dirichlet(np.full(nc, cfg.dirichlet_alpha))
        comp = g.choice(nc, size=L, p=w)
    else:
        comp = g.integers(0, nc, size=L)
    eps = g.standard_normal((L, d), dtype=np.float32)
    eps *= sd[comp]
    eps += mu[comp]
    return eps


def _head_queries_f32(cfg: LayerConfig, head: int) -> np.ndarray:
    L, d = cfg.L, cfg.d
    g = _rng(cfg, head, 0)
    u = g.standard_normal((cfg.q_directions, d), dtype=np.float32)
    u /= np.linalg.norm(u, axis=1, keepdims=True)
    j = g.integers(0, cfg.q_directions, size=L)
    x = g.standard_normal((L, d), dtype=np.float32)
    x *= np.float32(0.2 / np.sqrt(d))
    x += u[j]
    x /= np.linalg.norm(x, axis=1, keepdims=True)
    r = g.lognormal(0.0, 0.7, size=(L, 1)).astype(np.float32)
    x *= r
    return x


def _head_values_f32(cfg: LayerConfig, head: int) -> np.ndarray:
    return _rng(cfg, head, 2).standard_normal((cfg.L, cfg.d), dtype=np.float32)


def make_head(cfg: LayerConfig, head: int, step: int = 0):
    """(Q, K, V) of one head as bf16 bit patterns, each [L, d] uint16."""
    out = []
    for role, fn in ((0, _head_queries_f32), (1, _head_keys_f32), (2, _head_values_f32)):
        x = fn(cfg, head)
        for s in range(1, step + 1):
            x += np.float32(0.02) * _rng(cfg, head, 10 + role, s).standard_normal(
                x.shape, dtype=np.float32)
        out.append(f32_to_bf16_bits(x))
    return tuple(out)


def make_layer(cfg: LayerConfig, step: int = 0, heads=None):
    """(Q, K, V) as bf16 bit patterns, each [B, H', L, d] uint16 (B must be 1
    for a head subset).  ``heads`` selects a subset of heads (default: all)."""
    hs = list(range(cfg.H)) if heads is None else list(heads)
    shape = (cfg.B, len(hs), cfg.L, cfg.d)
    Q = np.empty(shape, np.uint16)
    K = np.empty(shape, np.uint16)
    V = np.empty(shape, np.uint16)
    for b in range(cfg.B):
        for i, h in enumerate(hs):
            hh = h + b * cfg.H
            Q[b, i], K[b, i], V[b, i] = make_head(cfg, hh, step)
    return Q, K, V


def _make_head_job(args):
    cfg, head, step = args
    return head, make_head(cfg, head, step)


def make_layer_parallel(cfg: LayerConfig, step: int = 0, procs: int | None = None):
    """make_layer for B = 1 with heads generated in a spawn-started process pool
    (bit-identical to make_layer; start it before the parent touches CUDA)."""
    import multiprocessing as mp
    import os
    assert cfg.B == 1
    procs = procs or min(32, os.cpu_count() or 1)
    shape = (1, cfg.H, cfg.L, cfg.d)
    Q, K, V = (np.empty(shape, np.uint16) for _ in range(3))
    with mp.get_context("spawn").Pool(procs) as pool:
        for h, (q, k, v) in pool.imap_unordered(_make_head_job, [(cfg, h, step) for h in range(cfg.H)]):
            Q[0, h], K[0, h], V[0, h] = q, k, v
    return Q, K, V
