"""N_max calibration over a stack of synthetic layers on the GPU (AdaCluster
Sec. 4.1: k_max is set so that the top 15% of layers run full attention),
with one context carried across the layers through ac_state_export/import.

1. Step 0 of every layer with an N_max too large to trigger: each unit's
   AC_T_FALLBACK_AT (the cluster count at the head of its last stage) is
   checked against the oracle's stage bookkeeping.
2. ac_calibrate_n_max picks N_max for a 15% dense share.
3. Every layer again with that N_max: exactly the units at or above it fall
   back, bit-exact against the oracle's Algorithm 1.
4. The one context, switched between layers by state import, runs each layer's
   warm step as a context dedicated to that layer does."""
import dataclasses

import numpy as np
import pytest

from _gpu_common import compare_layer, dev, gpu_state, host_f32
from oracle import oracle as orc
from cluster_routed_sparse_b200 import _lib as L_
from cluster_routed_sparse_b200 import synth
from cluster_routed_sparse_b200.api import SparseLayer, calibrate_n_max

pytestmark = pytest.mark.gpu

BASE = synth.LayerConfig("stack-L4096-H2-d64", 1, 2, 4096, 64, Cq=16, m0=32, n_max=6000,
                         tau_mode=synth.TAU_ABSOLUTE, tau_value=4.0, topk=8, iters_q=5, iters_k=5)
# layers of decreasing compactness: more mixture components per head, one absolute tau
# for the stack (App. A.5 uses absolute thresholds)
STACK = [dataclasses.replace(BASE, name=f"stack-layer{i}", key_components=nc, seed=BASE.seed + 97 * i)
         for i, nc in enumerate([16, 48, 100, 200, 300, 400])]


def _ctx(cfg, n_max):
    return SparseLayer(1, cfg.H, cfg.L, cfg.d, Cq=cfg.Cq, m0=cfg.m0, n_max=n_max, tau_mode=cfg.tau_mode,
                       tau_value=cfg.tau_value, topk=cfg.topk, iters_q=cfg.iters_q, iters_k=cfg.iters_k,
                       iters_warm=cfg.iters_warm, seed=5)


def _oracle_fallback_at(kc, m0, L, rule):
    out = []
    for h in range(kc.n_k.shape[0]):
        if kc.F[h]:
            out.append(int(kc.n_k[h]))
            continue
        T, nU, tot = int(kc.stages[h]), L, 0
        for t in range(T - 1):
            tot += orc.stage_clusters(m0, nU, L, t, rule)
            nU -= int((kc.removed_stage[h] == t).sum())
        out.append(tot)
    return out


def test_layer_stack_calibration_and_state_across_layers():
    data = [synth.make_layer(cfg) for cfg in STACK]
    big = _ctx(BASE, BASE.n_max)  # one context for the whole stack, n_max too large to trigger
    f_all, states = [], []
    for cfg, (Q, K, V) in zip(STACK, data):
        big.forward(dev(Q), dev(K), dev(V))
        big.synchronize()
        f = big.tensor(L_.AC_T_FALLBACK_AT).cpu().numpy().tolist()
        assert not big.tensor(L_.AC_T_DENSE).cpu().numpy().any()
        p = orc.Params.from_layer_config(cfg, seed=5)
        kc = orc.cluster_k_multistage(K[0], p)
        assert f == _oracle_fallback_at(kc, cfg.m0, cfg.L, cfg.stage_rule), cfg.name
        f_all += f
        states.append(big.export_state())
    n_max = calibrate_n_max(f_all, 0.15)
    k = int(np.ceil(0.15 * len(f_all)))
    assert sum(v >= n_max for v in f_all) >= k and sorted(f_all, reverse=True)[k - 1] == n_max
    # every layer again with the calibrated N_max: bit-exact against the oracle
    dense_units = 0
    for i, (cfg, (Q, K, V)) in enumerate(zip(STACK, data)):
        c2 = dataclasses.replace(cfg, n_max=n_max)
        p = orc.Params.from_layer_config(c2, seed=5)
        lay = _ctx(c2, n_max)
        O = lay.forward(dev(Q), dev(K), dev(V))
        lay.synchronize()
        gs = gpu_state(lay)
        r = orc.layer(Q[0], K[0], V[0], p, rows=np.arange(0, cfg.L, 61))
        compare_layer(gs, r, p)
        np.testing.assert_array_equal(gs["dense"], [1 if v >= n_max else 0 for v in f_all[2 * i:2 * i + 2]])
        dense_units += int(gs["dense"].sum())
        Os = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)[:, ::61]
        for h in range(cfg.H):
            d_ = Os[h] - r.O[h]
            assert np.abs(d_).max() <= 2e-2 and np.linalg.norm(d_) <= 5e-3 * np.linalg.norm(r.O[h])
        lay.close()
    assert dense_units == sum(v >= n_max for v in f_all)
    # the shared context, switched between layers by state import, gives each layer's warm step
    for i, (cfg, (Q, K, V)) in enumerate(zip(STACK, data)):
        big.import_state(states[i])
        ref = _ctx(BASE, BASE.n_max)
        ref.forward(dev(Q), dev(K), dev(V))
        Oref = ref.forward(dev(Q), dev(K), dev(V), warm=True)
        Ob = big.forward(dev(Q), dev(K), dev(V), warm=True)
        big.synchronize()
        ref.synchronize()
        np.testing.assert_array_equal(host_f32(Ob), host_f32(Oref), err_msg=cfg.name)
        ref.close()
    big.close()
