"""The pooled tau when the heads of one layer are split over ranks (AdaCluster
Sec. 4.1: tau from the stage-0 distances of the whole layer), on CPU with two
gloo ranks (127.0.0.1).

Each rank holds the stage-0 distances of its own heads and reduces them the
way the step-0 clustering does (fixed-point sum and count for the mean rule;
8-bit digit histograms for the percentile rule, here in numpy); the partial
results cross the ranks through the binding's torch.distributed exchange
function, and the library's host steps (ac_tau_mean_from_sums,
ac_tau_radix_pick) finish tau.  Every rank must get the tau the oracle computes
over all distances together, bit for bit."""
import os
import socket
import sys

import numpy as np
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _distances(rank):
    g = np.random.default_rng(100 + rank)
    n = 5000 + 1234 * rank  # ranks hold different numbers of keys
    d = g.lognormal(0.5, 0.6, n).astype(np.float32)
    d[:7] = d[7]  # ties
    return d


def _rank(rank, world, port, out):
    sys.path.insert(0, ROOT)
    from cluster_routed_sparse_b200 import api
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        xchg = api.tau_exchange_allreduce()
        d = _distances(rank)
        res = {}
        # mean rule: {sum floor(d 2^24), n}
        v = np.array([int((d.astype(np.float64) * 16777216.0).astype(np.uint64).sum()), d.size], np.uint64)
        xchg(v)
        res["mean"] = api.tau_mean_from_sums(1.5, int(v[0]), int(v[1]))
        # percentile rule: {n}, then four digit histograms
        for permille in (900, 1, 1000, 503):
            n = np.array([d.size], np.uint64)
            xchg(n)
            idx = min(max((permille * int(n[0]) + 999) // 1000 - 1, 0), int(n[0]) - 1)
            state = [0, 0, idx]
            bits = d.view(np.uint32)
            for shift in (24, 16, 8, 0):
                m = (bits & np.uint32(state[1])) == np.uint32(state[0])
                hist = np.bincount((bits[m] >> np.uint32(shift)) & np.uint32(255), minlength=256).astype(np.uint64)
                xchg(hist)
                state = api.tau_radix_pick(hist, shift, state)
            res[permille] = float(np.array([state[0]], np.uint32).view(np.float32)[0])
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_pooled_tau_over_two_ranks_equals_the_oracle():
    from oracle import oracle as orc
    world = 2
    port = _free_port()
    with mp.Manager() as m:
        out = m.dict()
        mp.spawn(_rank, args=(world, port, out), nprocs=world, join=True)
        res = dict(out)
    alld = np.concatenate([_distances(r) for r in range(world)])
    want = {"mean": orc.tau(alld, orc.TAU_MEAN_FACTOR, 1.5)}
    for permille in (900, 1, 1000, 503):
        want[permille] = orc.tau(alld, orc.TAU_PERCENTILE, float(permille))
    for r in range(world):
        for key, w in want.items():
            assert np.float32(res[r][key]) == np.float32(w), (r, key, res[r][key], w)


def test_host_steps_reject_bad_input():
    sys.path.insert(0, ROOT)
    import pytest
    from cluster_routed_sparse_b200 import api, _lib
    with pytest.raises(_lib.ACError):
        api.tau_mean_from_sums(1.5, 10, 0)
    with pytest.raises(_lib.ACError):
        api.tau_radix_pick([1] * 256, 12, [0, 0, 0])   # not a digit boundary
    with pytest.raises(_lib.ACError):
        api.tau_radix_pick([0] * 256, 24, [0, 0, 0])   # empty histogram: no rank 0
