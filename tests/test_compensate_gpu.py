"""Centroid compensation of the unselected key clusters on the GPU
(ClusterAttention Sec. 1.2, Eq. (5)-(6)): every unselected non-empty key
cluster enters each query's softmax as one pseudo-key, its member mean k,
carrying its member-mean value v and the weight |c| exp(q . k / sqrt(d)).

Against the oracle's attention_rows_comp (fp64) at the attention tolerance;
the clustering and the selections stay bit-exact, as without compensation."""
import dataclasses

import numpy as np
import pytest

from _gpu_common import compare_layer, dev, gpu_state, host_f32, make_layer_ctx
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth

pytestmark = pytest.mark.gpu

CASES = [synth.CONFIGS[1],
         synth.LayerConfig("comp-L6000-H3-d128", 1, 3, 6000, 128, Cq=20, m0=40, n_max=160,
                           tau_mode=synth.TAU_MEAN_FACTOR, tau_value=1.0, topk=-100, key_components=90,
                           iters_q=4, iters_k=4, diffuse_heads=(2,)),
         synth.LayerConfig("comp-heavy-L3000-H2-d64", 1, 2, 3000, 64, Cq=8, m0=24, n_max=96,
                           tau_mode=synth.TAU_MEAN_FACTOR, tau_value=1.0, topk=-200, key_components=60,
                           dirichlet_alpha=0.3)]


@pytest.mark.parametrize("cfg", CASES, ids=[c.name for c in CASES])
def test_compensated_layer_matches_oracle(cfg):
    Q, K, V = synth.make_layer(cfg)
    p = dataclasses.replace(orc.Params.from_layer_config(cfg, seed=17), compensate=1)
    lay = make_layer_ctx(p, cfg.B, cfg.H, cfg.L, cfg.d)
    O = lay.forward(dev(Q), dev(K), dev(V))
    lay.synchronize()
    gs = gpu_state(lay)
    r = orc.layer(Q[0], K[0], V[0], p)
    compare_layer(gs, r, p, O_gpu=host_f32(O).reshape(cfg.H, cfg.L, cfg.d))
    # compensation changes the output of the sparse heads (it is not a no-op)
    p0 = dataclasses.replace(p, compensate=0)
    r0 = orc.layer(Q[0], K[0], V[0], p0, rows=np.arange(0, cfg.L, 97))
    Oc = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)[:, ::97]
    for h in range(cfg.H):
        if not r.kc.F[h]:
            assert np.abs(Oc[h] - r0.O[h]).max() > 1e-2
    # a warm step with compensation
    O2 = lay.forward(dev(Q), dev(K), dev(V), warm=True)
    lay.synchronize()
    rw = orc.layer(Q[0], K[0], V[0], p, warm_from=r)
    compare_layer(gpu_state(lay), rw, p, O_gpu=host_f32(O2).reshape(cfg.H, cfg.L, cfg.d), check_step0=False)
    lay.close()
