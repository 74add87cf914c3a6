"""One layer's heads split over two contexts, tau pooled through the exchange
function (ac_set_tau_exchange), against one context over all heads: every
output must be bit-identical (AdaCluster Sec. 4.1: tau from the stage-0
distances of the whole layer; Algorithm 1 is otherwise per head).

The two contexts stand in for two ranks on one GPU: each runs in its own host
thread and stream, and their exchange meets on the host (a barrier and a sum),
so no kernel of one waits for the other's."""
import threading

import numpy as np
import pytest
import torch

from _gpu_common import dev, gpu_state, host_f32
from cluster_routed_sparse_b200 import synth
from cluster_routed_sparse_b200.api import SparseLayer

pytestmark = pytest.mark.gpu


class HostSum:
    """Sum of the contexts' partial results, met on a host barrier."""

    def __init__(self, n):
        self.n, self.bar, self.buf, self.calls = n, threading.Barrier(n, timeout=120), {}, 0

    def fn(self, idx):
        def f(vals):
            self.buf[idx] = vals.copy()
            self.bar.wait()
            tot = sum(self.buf[i].astype(np.uint64) for i in range(self.n))
            self.bar.wait()
            if idx == 0:
                self.calls += 1
            vals[:] = tot
        return f


def _layer(cfg, H, unit0):
    return SparseLayer(1, H, cfg.L, cfg.d, Cq=cfg.Cq, m0=cfg.m0, n_max=cfg.n_max, tau_mode=cfg.tau_mode,
                       tau_value=cfg.tau_value, topk=cfg.topk, iters_q=cfg.iters_q, iters_k=cfg.iters_k,
                       iters_warm=cfg.iters_warm, seed=99, unit0=unit0)


CASES = [synth.LayerConfig("split-mean-L4096-H4-d64", 1, 4, 4096, 64, Cq=16, m0=32, n_max=128,
                           tau_mode=synth.TAU_MEAN_FACTOR, tau_value=1.0, topk=8, key_components=48,
                           diffuse_heads=(3,)),
         synth.LayerConfig("split-p80-L3000-H5-d128", 1, 5, 3000, 128, Cq=12, m0=24, n_max=96,
                           tau_mode=synth.TAU_PERCENTILE, tau_value=800.0, topk=-150, key_components=40)]
KEYS = ("labels_q", "cent_q", "labels_k", "cent_k", "n_k", "dense", "stages", "removed_stage", "counts_k", "sel",
        "ksel", "comp", "kmax", "kmin")


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_split_heads_with_pooled_tau_is_bit_identical(cfg):
    Q, K, V = synth.make_layer(cfg)
    whole = _layer(cfg, cfg.H, 0)
    O_whole = whole.forward(dev(Q), dev(K), dev(V))
    whole.synchronize()
    ref = gpu_state(whole)
    ref_O = host_f32(O_whole)
    O_whole_warm = whole.forward(dev(Q), dev(K), dev(V), warm=True)
    whole.synchronize()
    ref_warm_O = host_f32(O_whole_warm)
    parts = [(0, 2), (2, cfg.H)]
    xs = HostSum(len(parts))
    res = [None] * len(parts)
    errors = []

    def run(i, lo, hi):
        try:
            s = torch.cuda.Stream()
            with torch.cuda.stream(s):
                lay = _layer(cfg, hi - lo, lo)
                lay.set_tau_exchange(xs.fn(i))
                q, k, v = (dev(x[:, lo:hi]) for x in (Q, K, V))
                O = lay.forward(q, k, v)
                lay.synchronize()
                st = gpu_state(lay)
                Ow = lay.forward(q, k, v, warm=True)
                lay.synchronize()
                res[i] = (st, host_f32(O), host_f32(Ow))
                lay.close()
        except Exception as exc:  # reported below
            errors.append(repr(exc))

    th = [threading.Thread(target=run, args=(i, lo, hi)) for i, (lo, hi) in enumerate(parts)]
    for t in th:
        t.start()
    for t in th:
        t.join(timeout=600)
    assert not errors, errors
    assert xs.calls == (1 if cfg.tau_mode == synth.TAU_MEAN_FACTOR else 5)
    for i, (lo, hi) in enumerate(parts):
        st, O, Ow = res[i]
        assert st["tau"][0] == ref["tau"][0]
        for key in KEYS:
            np.testing.assert_array_equal(st[key], ref[key][lo:hi], err_msg=f"{key}, heads {lo}-{hi}")
        np.testing.assert_array_equal(O, ref_O[:, lo:hi], err_msg="step-0 output")
        np.testing.assert_array_equal(Ow, ref_warm_O[:, lo:hi], err_msg="warm-step output")
    whole.close()
