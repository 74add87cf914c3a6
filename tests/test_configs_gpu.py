"""GPU parity on the layer shapes of every workload, end to end against the
oracle (not in lockstep):

* CogVideoX-2B-class (B=1, H=30, L=17,550, d=64): the whole layer against the
  oracle on all heads; the two diffuse heads reach N_max = 600 and run dense
  (AdaCluster Algorithm 1 lines 7-9, Algorithm 3 line 6).
* Wan-2.1-1.3B-class (H=12, L=32,760, d=128): the percentile rule for tau over
  all heads, and the top-k at 5 %, 10 % and 20 % of the key clusters.
* Wan-2.1-14B-class (H=40, L=75,600, d=128): step 0 and a warm step on
  sampled heads, each run by the oracle on its own with the layer's seeds and
  the GPU's pooled tau, so that the centre updates of clusters with thousands
  of members, the stage loop and the final assignment at full size are
  compared, not only re-assigned.
* Long heavy-tailed (H=24, L=118,800, Dirichlet(0.3) component weights):
  sampled heads as above; most key clusters end in partly filled 8-row groups.
* A dense unit that walks more key ranges than the attention kernel caches in
  shared memory, and the AvgClus ablation (one stage, tau = +inf)."""
import dataclasses
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

from _gpu_common import assert_attention, compare_layer, dev, gpu_state, host_f32, make_layer_ctx
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth

pytestmark = pytest.mark.gpu

PER_UNIT = ("labels_q", "cent_q", "counts_q", "perm_q", "offs_q", "labels_k", "dmin_k", "cent_k", "n_k", "dense",
            "counts_k", "sse", "comp", "mse", "perm_k", "offs_k", "score", "sel", "ksel", "stages",
            "removed_stage", "kmax", "kmin")


def _unit(gs, h):
    out = {k: (v[h:h + 1] if k in PER_UNIT else v) for k, v in gs.items()}
    return out


def _rows(gs, h, L, n_spread=48, n_tails=24):
    """Query rows spread over the sequence plus the last rows of the query clusters."""
    offs = gs["offs_q"][h]
    tails = gs["perm_q"][h][np.maximum(offs[1:] - 1, 0)]
    tails = tails[np.diff(offs) > 0][:n_tails]
    return np.unique(np.concatenate([np.linspace(0, L - 1, n_spread).astype(np.int64), tails]))


def _check_attention(Q, K, V, O, gs, r, heads, L, what, sel=None):
    for i, h in enumerate(heads):
        rows = _rows(gs, h, L)
        s = (r.sel[i] if sel is None else sel[i])
        ref = orc.attention_rows(Q[0, h], K[0, h], V[0, h], r.labels_q[i], r.kc.labels[i], s,
                                 bool(r.kc.F[i]), rows)
        assert_attention(O[h][rows], ref, f"{what} attention h{h}")


def _oracle_heads(Q, K, V, p, heads, tau, warm_from=None):
    """Each head alone with the layer's seeds (unit0 = head) and the GPU's pooled
    tau as an absolute threshold; heads run in parallel threads."""
    def one(i_h):
        i, h = i_h
        ph = dataclasses.replace(p, tau_mode=orc.TAU_ABSOLUTE, tau_value=float(tau), unit0=h)
        wf = None if warm_from is None else warm_from[i]
        return orc.layer(Q[0, h:h + 1], K[0, h:h + 1], V[0, h:h + 1], ph, warm_from=wf, attention=False)
    with ThreadPoolExecutor(max(1, len(heads))) as ex:
        return list(ex.map(one, enumerate(heads)))


def test_cogvideox_class_layer_with_dense_heads():
    cfg = synth.CONFIGS[2]
    Q, K, V = synth.make_layer_parallel(cfg)
    p = orc.Params.from_layer_config(cfg, seed=1234)
    lay = make_layer_ctx(p, 1, cfg.H, cfg.L, cfg.d)
    O = lay.forward(dev(Q), dev(K), dev(V))
    lay.synchronize()
    gs = gpu_state(lay)
    r = orc.layer(Q[0], K[0], V[0], p, attention=False)
    compare_layer(gs, r, p)
    assert list(np.nonzero(gs["dense"])[0]) == list(cfg.diffuse_heads), gs["dense"]
    assert (gs["n_k"][list(cfg.diffuse_heads)] >= cfg.n_max).all()
    Oh = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)
    heads = [0, 1, 7, 29]
    sub = dataclasses.replace(r, labels_q=r.labels_q[heads], kc=dataclasses.replace(
        r.kc, labels=r.kc.labels[heads], F=r.kc.F[heads]), sel=[r.sel[h] for h in heads])
    _check_attention(Q, K, V, Oh, gs, sub, heads, cfg.L, "cogvideox")
    lay.close()


def test_wan13b_class_layer_percentile_tau_and_topk_sweep():
    cfg = synth.CONFIGS[3]
    Q, K, V = synth.make_layer_parallel(cfg)
    p = orc.Params.from_layer_config(cfg, seed=1234)
    lay = make_layer_ctx(p, 1, cfg.H, cfg.L, cfg.d)
    q, k, v = dev(Q), dev(K), dev(V)
    O = lay.forward(q, k, v)
    lay.synchronize()
    gs = gpu_state(lay)
    r = orc.layer(Q[0], K[0], V[0], p, attention=False)
    compare_layer(gs, r, p)  # tau at the 90th percentile of the pooled stage-0 distances, bit-exact
    heads = [0, 5, 11]
    Oh = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)
    sub = dataclasses.replace(r, labels_q=r.labels_q[heads], kc=dataclasses.replace(
        r.kc, labels=r.kc.labels[heads], F=r.kc.F[heads]), sel=[r.sel[h] for h in heads])
    _check_attention(Q, K, V, Oh, gs, sub, heads, cfg.L, "wan1.3b top-k 10%")
    for topk in (-50, -200):
        lay.score_select(topk)
        O2 = lay.sparse_attn(q, k, v)
        lay.synchronize()
        gs2 = gpu_state(lay)
        _, sel, kk = orc.score_select(r.Cq, r.st, r.kc.n_k, topk)
        np.testing.assert_array_equal(gs2["ksel"], kk)
        for h in range(cfg.H):
            np.testing.assert_array_equal(gs2["sel"][h, :, :kk[h]], sel[h], err_msg=f"top-k {topk} h{h}")
        _check_attention(Q, K, V, host_f32(O2).reshape(cfg.H, cfg.L, cfg.d), gs2, sub, heads, cfg.L,
                         f"wan1.3b top-k {-topk / 10}%", sel=[sel[h] for h in heads])
    lay.close()


def _sampled_heads_end_to_end(cfg, heads, warm: bool):
    Q, K, V = synth.make_layer_parallel(cfg)
    p = orc.Params.from_layer_config(cfg, seed=1234)
    lay = make_layer_ctx(p, 1, cfg.H, cfg.L, cfg.d)
    q, k, v = dev(Q), dev(K), dev(V)
    O = lay.forward(q, k, v)
    lay.synchronize()
    gs = gpu_state(lay)
    tau = float(gs["tau"][0])
    rs = _oracle_heads(Q, K, V, p, heads, tau)
    Oh = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)
    for h, r in zip(heads, rs):
        compare_layer(_unit(gs, h), r, dataclasses.replace(p, tau_mode=orc.TAU_ABSOLUTE, tau_value=tau))
        _check_attention(Q, K, V, Oh, gs, r, [h], cfg.L, f"{cfg.name} step 0")
    if warm:
        O = lay.forward(q, k, v, warm=True)
        lay.synchronize()
        gs = gpu_state(lay)
        rw = _oracle_heads(Q, K, V, p, heads, tau, warm_from=rs)
        Oh = host_f32(O).reshape(cfg.H, cfg.L, cfg.d)
        for h, r in zip(heads, rw):
            compare_layer(_unit(gs, h), r, p, check_step0=False)
            _check_attention(Q, K, V, Oh, gs, r, [h], cfg.L, f"{cfg.name} warm step")
    lay.close()
    return gs


def test_wan14b_class_sampled_heads_end_to_end():
    gs = _sampled_heads_end_to_end(synth.CONFIGS[4], [3, 26], warm=True)
    assert not gs["dense"].any()


def test_long_heavy_tailed_sampled_heads_end_to_end():
    cfg = synth.CONFIGS[5]
    gs = _sampled_heads_end_to_end(cfg, [2, 19], warm=False)
    # heavy tails: clusters of fewer than 8 keys exist, i.e. partly filled 8-row groups of their own
    assert any((gs["counts_k"][h, :gs["n_k"][h]] < 8).any() for h in range(cfg.H))


def test_dense_unit_beyond_the_range_cache():
    """A dense unit with more non-empty key clusters (2,400) than the attention
    kernel keeps in shared memory (2,048): its key ranges are read from global
    memory.  tau = 0 absorbs no key, so the unit falls back after stage 0."""
    cfg = synth.LayerConfig("ranges-L8192-H1-d128", 1, 1, 8192, 128, Cq=8, m0=2400, n_max=2000,
                            tau_mode=synth.TAU_ABSOLUTE, tau_value=0.0, topk=4, iters_q=3, iters_k=3,
                            diffuse_heads=(0,))
    Q, K, V = synth.make_layer(cfg)
    p = orc.Params.from_layer_config(cfg, seed=3)
    lay = make_layer_ctx(p, 1, 1, cfg.L, cfg.d)
    O = lay.forward(dev(Q), dev(K), dev(V))
    lay.synchronize()
    gs = gpu_state(lay)
    r = orc.layer(Q[0], K[0], V[0], p, attention=False)
    compare_layer(gs, r, p)
    assert gs["dense"][0] == 1 and (gs["counts_k"][0, :gs["n_k"][0]] > 0).sum() > 2048
    _check_attention(Q, K, V, host_f32(O).reshape(1, cfg.L, cfg.d), gs, r, [0], cfg.L, "dense, uncached ranges")
    lay.close()


def test_avgclus_single_stage_ablation():
    """AvgClus (AdaCluster Sec. 4.4 Table 3): the same cluster count everywhere,
    i.e. one stage of Algorithm 1 with tau = +inf absorbing every key."""
    cfg = dataclasses.replace(synth.CONFIGS[1], tau_mode=synth.TAU_ABSOLUTE, tau_value=float("inf"))
    Q, K, V = synth.make_layer(cfg)
    p = orc.Params.from_layer_config(cfg, seed=77)
    lay = make_layer_ctx(p, 1, cfg.H, cfg.L, cfg.d)
    O = lay.forward(dev(Q), dev(K), dev(V))
    lay.synchronize()
    gs = gpu_state(lay)
    r = orc.layer(Q[0], K[0], V[0], p)
    compare_layer(gs, r, p, O_gpu=host_f32(O).reshape(cfg.H, cfg.L, cfg.d))
    assert (gs["stages"] == 1).all() and (gs["n_k"] == cfg.m0).all() and not gs["dense"].any()
    lay.close()
