"""Parity at the bench workload (Wan-2.1-14B-class layer: B=1, H=40,
L=75,600, d=128) in the launch configuration bench.py times.  The whole layer
runs on the GPU; the oracle checks sampled heads and rows one by one, in
lockstep with the GPU's own centres, plus size-independent invariants on
every head."""
import numpy as np
import pytest

from _gpu_common import assert_attention, dev, gpu_state, host_f32, make_layer_ctx
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth

pytestmark = pytest.mark.gpu

HEADS = (0, 17, 39)


@pytest.fixture(scope="module")
def inputs():
    cfg = synth.CONFIGS[4]
    return cfg, synth.make_layer_parallel(cfg)


def _check_state(cfg, Q, K, V, O, gs, p, step0: bool):
    H, L = cfg.H, cfg.L
    # size-independent invariants on every head
    for h in range(H):
        nk = int(gs["n_k"][h])
        lab = gs["labels_k"][h]
        assert lab.min() >= 0 and lab.max() < nk
        np.testing.assert_array_equal(gs["perm_k"][h], np.argsort(lab, kind="stable"))
        np.testing.assert_array_equal(gs["perm_q"][h], np.argsort(gs["labels_q"][h], kind="stable"))
        np.testing.assert_array_equal(gs["counts_k"][h, :nk], np.bincount(lab, minlength=nk))
        if step0:
            rs = gs["removed_stage"][h]
            tot, nU = 0, L
            for t in range(int(gs["stages"][h])):
                m = orc.stage_clusters(cfg.m0, nU, L, t, p.stage_rule)
                tot += m
                nU -= int((rs == t).sum())
            assert tot == nk
            assert bool((rs < 0).any()) == bool(gs["dense"][h])
    for h in HEADS:
        nk = int(gs["n_k"][h])
        # query assignment against the GPU's centres (lockstep)
        _, xh = orc.qnorm(Q[0, h])
        lab_q, _ = orc.assign(xh, gs["cent_q"][h])
        np.testing.assert_array_equal(gs["labels_q"][h], lab_q, err_msg=f"query labels h{h}")
        # key assignment (Algorithm 1 line 22 / warm Lloyd) against the GPU's centres
        Kf = synth.bf16_bits_to_f32(K[0, h])
        lab_k, dm = orc.assign(Kf, gs["cent_k"][h, :nk])
        np.testing.assert_array_equal(gs["labels_k"][h], lab_k, err_msg=f"key labels h{h}")
        np.testing.assert_array_equal(gs["dmin_k"][h], dm)
        # stats and selection from the GPU's clusters
        kc = orc.KClusters(gs["labels_k"][h:h + 1], gs["cent_k"][h:h + 1], gs["n_k"][h:h + 1],
                           gs["dense"][h:h + 1], 0.0, None, None, None)
        st = orc.key_stats(K[0, h:h + 1], kc)
        np.testing.assert_array_equal(gs["counts_k"][h, :nk], st.counts[0, :nk])
        np.testing.assert_array_equal(gs["kmax"][h, :nk], st.kmax[0, :nk])
        np.testing.assert_array_equal(gs["kmin"][h, :nk], st.kmin[0, :nk])
        np.testing.assert_array_equal(gs["sse"][h, :nk], st.sse[0, :nk])
        _, sel, k = orc.score_select(gs["cent_q"][h:h + 1], st, gs["n_k"][h:h + 1], p.topk)
        assert gs["ksel"][h] == k[0]
        np.testing.assert_array_equal(gs["sel"][h, :, :k[0]], sel[0], err_msg=f"selection h{h}")
        # attention rows: spread over the sequence plus the last rows of clusters
        offs = gs["offs_q"][h]
        tails = gs["perm_q"][h][np.maximum(offs[1:] - 1, 0)][:32]
        rows = np.unique(np.concatenate([np.linspace(0, L - 1, 64).astype(np.int64), tails]))
        ref = orc.attention_rows(Q[0, h], K[0, h], V[0, h], gs["labels_q"][h], gs["labels_k"][h],
                                 sel[0], bool(gs["dense"][h]), rows)
        assert_attention(O[h][rows], ref, f"attention h{h}")


def test_wan14b_layer_step0_and_warm(inputs):
    cfg, (Q, K, V) = inputs
    p = orc.Params.from_layer_config(cfg, seed=1234)
    lay = make_layer_ctx(p, 1, cfg.H, cfg.L, cfg.d)
    q, k, v = dev(Q), dev(K), dev(V)
    for warm in (False, True):
        O = lay.forward(q, k, v, warm=warm)
        lay.synchronize()
        gs = gpu_state(lay)
        _check_state(cfg, Q, K, V, host_f32(O).reshape(cfg.H, cfg.L, cfg.d), gs, p, step0=not warm)
        assert not gs["dense"].any() or warm  # 500 planted components: no head falls back
    lay.close()
