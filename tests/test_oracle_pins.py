"""Pins of the CPU oracle against things other than itself.

Each test ties one oracle step to a hand-worked example (tests/golden/), a
published generator, a library routine (scikit-learn's Lloyd, torch SDPA), a
closed form or an invariant of the method on the AdaCluster pages
(arXiv 2604.18348) and the ClusterAttention error split.
"""
import ctypes
import json
import os

import numpy as np
import pytest

from conftest import GOLDEN
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def bf(x):
    return synth.f32_to_bf16_bits(np.asarray(x, np.float32))


# ----------------------------------------------------------------- generator

def test_splitmix64_published_vectors():
    g = _golden("splitmix64_vectors.json")
    lib = orc.lib()
    lib.or_splitmix64.restype = ctypes.c_uint64
    lib.or_splitmix64.argtypes = [ctypes.c_uint64, ctypes.c_int64]
    got0 = ["%016x" % lib.or_splitmix64(0, i) for i in range(3)]
    assert got0 == g["state_0_hex"]
    got1 = [lib.or_splitmix64(1234567, i) for i in range(5)]
    assert got1 == g["state_1234567"]


@pytest.mark.parametrize("n,m", [(1, 1), (7, 7), (10, 3), (4096, 16), (75600, 256), (5, 2)])
def test_seed_pick_strata(n, m):
    pos = orc.seed_pick(99, 3, 5, n, m)
    assert len(set(pos.tolist())) == m
    for j, p in enumerate(pos):
        assert (j * n) // m <= p < ((j + 1) * n) // m
    if m == n:
        assert (pos == np.arange(n)).all()


# ----------------------------------------------------------------- Sec. 3.1

def test_qnorm_against_fp64_norm():
    rng = np.random.default_rng(0)
    q = bf(rng.standard_normal((257, 64)) * rng.lognormal(0, 1, (257, 1)))
    q[5] = 0
    inv, xh = orc.qnorm(q)
    qf = synth.bf16_bits_to_f32(q).astype(np.float64)
    n = np.linalg.norm(qf, axis=1)
    ok = n > 0
    assert np.allclose(inv[ok] * n[ok], 1.0, rtol=0, atol=3e-7)
    assert inv[5] == 0 and (xh[5] == 0).all()
    assert np.allclose(np.linalg.norm(xh[ok].astype(np.float64), axis=1), 1.0, atol=1e-6)


def test_angular_clustering_scale_invariance():
    """Check (e): rescaling a query by a positive factor leaves its direction,
    hence the angular clustering, unchanged (App. A.2).  Powers of two scale
    bf16 exactly, so labels and centres must be bit-identical."""
    cfg = synth.CONFIGS[1]
    Q, _, _ = synth.make_layer(cfg, heads=[0])
    p = orc.Params.from_layer_config(cfg)
    lab0, C0, _ = orc.cluster_q(Q[0], p)
    rng = np.random.default_rng(1)
    e = rng.integers(-3, 4, size=(cfg.L, 1)).astype(np.float32)
    Qs = bf(synth.bf16_bits_to_f32(Q[0, 0]) * np.exp2(e))[None]
    lab1, C1, _ = orc.cluster_q(Qs, p)
    assert (lab0 == lab1).all()
    assert np.array_equal(C0, C1)


def test_angular_clustering_arbitrary_scale_near_invariant():
    """Check (e) with arbitrary factors in [0.1, 10]: the bf16 rounding of the
    rescaled query moves its direction by about 2^-9, so one assignment to the
    same centres agrees except on rows whose best/second gap is that small."""
    cfg = synth.CONFIGS[1]
    Q, _, _ = synth.make_layer(cfg, heads=[1])
    p = orc.Params.from_layer_config(cfg)
    _, C0, _ = orc.cluster_q(Q[0], p)
    rng = np.random.default_rng(2)
    s = rng.uniform(0.1, 10, size=(cfg.L, 1)).astype(np.float32)
    Qs = bf(synth.bf16_bits_to_f32(Q[0, 0]) * s)
    x0 = orc.qnorm(Q[0, 0])[1]
    x1 = orc.qnorm(Qs)[1]
    lab0, _ = orc.assign(x0, C0[0])
    lab1, _ = orc.assign(x1, C0[0])
    D = ((x0[:, None, :].astype(np.float64) - C0[0][None].astype(np.float64)) ** 2).sum(-1)
    srt = np.sort(D, axis=1)
    near = (srt[:, 1] - srt[:, 0]) < 2e-2
    assert (lab0[~near] == lab1[~near]).all()
    assert (lab0 != lab1).mean() < 0.01


# ----------------------------------------------------------------- k-means

def test_assign_bruteforce_fp64():
    rng = np.random.default_rng(3)
    X = rng.standard_normal((500, 16)).astype(np.float32)
    C = rng.standard_normal((37, 16)).astype(np.float32)
    C[9] = C[4]  # exact duplicate: ties go to the lower id
    lab, dm = orc.assign(X, C)
    D = ((X[:, None, :].astype(np.float64) - C[None].astype(np.float64)) ** 2).sum(-1)
    srt = np.sort(D, axis=1)
    clear = (srt[:, 1] - srt[:, 0]) > 1e-5 * srt[:, 0]
    assert (lab[clear] == D[clear].argmin(1)).all()
    assert np.allclose(dm, D[np.arange(500), lab], rtol=1e-5)
    assert not (lab == 9).any()


def test_update_is_member_mean_and_keeps_empty():
    rng = np.random.default_rng(4)
    X = rng.standard_normal((300, 8)).astype(np.float32)
    lab = rng.integers(0, 5, 300).astype(np.int32)
    lab[lab == 3] = 2  # cluster 3 empty
    C0 = rng.standard_normal((5, 8)).astype(np.float32)
    C, cnt = orc.update(X, lab, C0)
    for c in range(5):
        if c == 3:
            assert cnt[c] == 0 and np.array_equal(C[c], C0[c])
        else:
            m = X[lab == c].astype(np.float64).mean(0)
            assert cnt[c] == (lab == c).sum()
            assert np.allclose(C[c], m, rtol=1e-5, atol=1e-6)


def test_kmeans_matches_sklearn_lloyd():
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(5)
    centres = rng.standard_normal((6, 5)) * 10
    X = (centres[rng.integers(0, 6, 600)] + rng.standard_normal((600, 5))).astype(np.float32)
    init = X[orc.seed_pick(7, 0, 0, 600, 6)]
    lab, dm, C = orc.kmeans(X, init, 8)
    km = KMeans(n_clusters=6, init=init.astype(np.float64), n_init=1, max_iter=8, tol=0.0,
                algorithm="lloyd").fit(X.astype(np.float64))
    assert (km.labels_ == lab).all()
    assert np.allclose(km.cluster_centers_, C, rtol=1e-5, atol=1e-5)


def test_lloyd_objective_monotone():
    """Check (b): J never increases across an assignment or an update."""
    cfg = synth.CONFIGS[1]
    Q, K, _ = synth.make_layer(cfg, heads=[0])
    for X in (synth.bf16_bits_to_f32(K[0, 0]), orc.qnorm(Q[0, 0])[1]):
        init = X[orc.seed_pick(11, 0, 0, X.shape[0], 24)]
        _, _, _, jt = orc.kmeans(X, init, 10, trace=True)
        assert (np.diff(jt) <= 1e-6 * jt[:-1]).all(), jt


def test_planted_partition_recovery():
    """Well-separated mixture (Sec. 3.2.2: stages continue until every token
    sits in a compact cluster): every multi-stage key cluster is pure."""
    rng = np.random.default_rng(6)
    L, d, nc = 2048, 16, 12
    mu = rng.standard_normal((nc, d)) * 8
    comp = rng.integers(0, nc, L)
    Kf = mu[comp] + 0.05 * rng.standard_normal((L, d))
    K16 = bf(Kf)[None]
    p = orc.Params(Cq=4, m0=8, n_max=200, tau_mode=orc.TAU_ABSOLUTE, tau_value=1.0, topk=2,
                   iters_k=10)
    kc = orc.cluster_k_multistage(K16, p)
    lab = kc.labels[0]
    for c in np.unique(lab):
        assert len(np.unique(comp[lab == c])) == 1
    assert kc.F[0] == 0


# ----------------------------------------------------------------- tau

def test_tau_rules_by_hand():
    d = np.arange(1, 11, dtype=np.float32)
    assert orc.tau(d, orc.TAU_PERCENTILE, 900) == 9.0     # nearest rank ceil(0.9*10) = 9
    assert orc.tau(d, orc.TAU_PERCENTILE, 1000) == 10.0
    assert orc.tau(d, orc.TAU_PERCENTILE, 1) == 1.0
    assert orc.tau(np.array([1, 2, 3], np.float32), orc.TAU_MEAN_FACTOR, 1.5) == 3.0
    assert orc.tau(d, orc.TAU_ABSOLUTE, 4.25) == 4.25
    rng = np.random.default_rng(7)
    x = rng.uniform(0, 20, 100000).astype(np.float32)
    assert abs(orc.tau(x, orc.TAU_MEAN_FACTOR, 1.5) - 1.5 * x.astype(np.float64).mean()) < 1e-5


# ----------------------------------------------------------------- Algorithm 1

@pytest.mark.parametrize("case", [0, 1, 2])
def test_multistage_hand_example(case):
    g = _golden("multistage_hand.json")
    c = g["cases"][case]
    K16 = bf(np.array(g["keys"], np.float32))[None]
    p = orc.Params(Cq=1, m0=g["m0"], n_max=c["n_max"], tau_mode=orc.TAU_ABSOLUTE,
                   tau_value=c["tau"], topk=1, iters_k=g["iters"], stage_rule=c["stage_rule"])
    kc = orc.cluster_k_multistage(K16, p)
    assert kc.n_k[0] == c["n_k"] and kc.F[0] == c["F"] and kc.stages[0] == c["stages"]
    assert kc.labels[0].tolist() == c["labels"]
    assert kc.removed_stage[0].tolist() == c["removed_stage"]
    assert np.allclose(kc.C[0, :c["n_k"]], np.array(c["centres"]), rtol=1e-6)
    r0 = np.array(c["removed_stage"]) == 0
    # fp32 centres of ~100-sized coordinates carry ~2^-24 * 100 absolute error
    assert np.allclose(kc.removed_dist[0][r0], np.array(g["stage0_distances"])[r0], rtol=0,
                       atol=1e-5)


def test_multistage_invariants_tiny_config():
    cfg = synth.CONFIGS[1]
    _, K, _ = synth.make_layer(cfg)
    p = orc.Params.from_layer_config(cfg)
    kc = orc.cluster_k_multistage(K[0], p)
    L = cfg.L
    # tau follows the pooled mean rule
    assert kc.tau > 0
    for h in range(cfg.H):
        nk, rs, rd = int(kc.n_k[h]), kc.removed_stage[h], kc.removed_dist[h]
        assert (kc.labels[h] >= 0).all() and (kc.labels[h] < nk).all()
        # every token that left U had d < tau at that stage
        assert (rd[rs >= 0] < kc.tau).all()
        # tokens only stay unabsorbed when the fallback fired
        assert ((rs < 0).any()) == bool(kc.F[h])
        # n_k is the sum of the stage sizes m_t
        tot, nU = 0, L
        for t in range(int(kc.stages[h])):
            m = orc.stage_clusters(cfg.m0, nU, L, t, p.stage_rule)
            tot += m
            nU -= int((rs == t).sum())
        assert tot == nk
    # recompute the stage-0 mean from the stage-0 distances is not possible
    # from outputs alone; check the rule on tokens absorbed at stage 0
    assert (kc.removed_dist[kc.removed_stage == 0] < kc.tau).all()


def test_multistage_infinite_tau_is_plain_kmeans():
    """tau = inf: stage 0 absorbs everything, so Algorithm 1 reduces to one
    k-means with m0 centres (seeded with tag 1) and its final assignment."""
    cfg = synth.CONFIGS[1]
    _, K, _ = synth.make_layer(cfg, heads=[0])
    p = orc.Params(Cq=4, m0=32, n_max=128, tau_mode=orc.TAU_ABSOLUTE, tau_value=np.inf,
                   topk=4, iters_k=10, seed=77)
    kc = orc.cluster_k_multistage(K[0], p)
    assert kc.n_k[0] == 32 and kc.F[0] == 0 and kc.stages[0] == 1
    X = synth.bf16_bits_to_f32(K[0, 0])
    init = X[orc.seed_pick(77, 0, 1, cfg.L, 32)]
    lab, _, C = orc.kmeans(X, init, 10)
    assert np.array_equal(kc.C[0, :32], C)
    assert (kc.labels[0] == lab).all()


def test_multistage_zero_tau_falls_back():
    """tau = 0 absorbs nothing (d < 0 never holds): every stage re-clusters all
    L tokens with m0 centres until |C| >= N_max, then F is set."""
    cfg = synth.CONFIGS[1]
    _, K, _ = synth.make_layer(cfg, heads=[0])
    p = orc.Params(Cq=4, m0=32, n_max=100, tau_mode=orc.TAU_ABSOLUTE, tau_value=0.0,
                   topk=4, iters_k=2)
    kc = orc.cluster_k_multistage(K[0], p)
    assert kc.F[0] == 1 and kc.n_k[0] == 128 and kc.stages[0] == 4
    assert (kc.removed_stage[0] == -1).all()


def test_multistage_nmax_below_m0_falls_back_after_stage0():
    cfg = synth.CONFIGS[1]
    _, K, _ = synth.make_layer(cfg, heads=[1])
    p = orc.Params(Cq=4, m0=32, n_max=16, tau_mode=orc.TAU_MEAN_FACTOR, tau_value=0.5,
                   topk=4, iters_k=3)
    kc = orc.cluster_k_multistage(K[0], p)
    assert kc.n_k[0] == 32 and kc.F[0] == 1 and kc.stages[0] == 1


def test_single_query_clusters_when_cq_equals_l():
    """Cq = L: the seeded init takes every token (strata of width 1) and each
    distinct query stays alone in its cluster."""
    rng = np.random.default_rng(8)
    Q = bf(rng.standard_normal((1, 64, 16)))
    p = orc.Params(Cq=64, m0=1, n_max=2, tau_mode=0, tau_value=1.0, topk=1, iters_q=3)
    lab, C, cnt = orc.cluster_q(Q, p)
    assert (lab[0] == np.arange(64)).all() and (cnt == 1).all()


# ----------------------------------------------------------------- stats

def test_key_stats_against_numpy():
    cfg = synth.CONFIGS[1]
    _, K, _ = synth.make_layer(cfg)
    p = orc.Params.from_layer_config(cfg)
    kc = orc.cluster_k_multistage(K[0], p)
    st = orc.key_stats(K[0], kc)
    for h in range(cfg.H):
        X = synth.bf16_bits_to_f32(K[0, h]).astype(np.float64)
        lab = kc.labels[h]
        assert st.counts[h].sum() == cfg.L
        sse_tot = 0.0
        for c in range(int(kc.n_k[h])):
            m = lab == c
            assert st.counts[h, c] == m.sum()
            if m.any():
                assert np.array_equal(st.kmax[h, c], X[m].max(0).astype(np.float32))
                assert np.array_equal(st.kmin[h, c], X[m].min(0).astype(np.float32))
                s = ((X[m] - kc.C[h, c].astype(np.float64)) ** 2).sum()
                assert abs(st.sse[h, c] - s) <= 1e-4 * max(s, 1e-3)
                sse_tot += s
        assert abs(st.mse[h] - sse_tot / cfg.L) <= 1e-4 * sse_tot / cfg.L
        assert st.comp[h] == np.float32(1.0) / st.mse[h]


# ----------------------------------------------------------------- Eq. (1)

def test_quest_hand_example():
    g = _golden("quest_attention_hand.json")["quest"]
    S = orc.quest(np.array([g["q"]], np.float32), np.array([g["kmax"]], np.float32),
                  np.array([g["kmin"]], np.float32), np.array([2], np.int32))
    assert S[0, 0] == g["quest"]
    # Eq. (2) as printed (k+ / k- of the bounds) is not Eq. (1)
    q = np.array(g["q"], np.float64)
    e2 = np.maximum(q, 0) @ np.maximum(g["kmax"], 0) + np.minimum(q, 0) @ np.minimum(g["kmin"], 0)
    assert e2 == g["eq2_as_printed_value"] != g["quest"]


def test_quest_is_upper_bound_and_tensor_form():
    """Check (c): Quest(q, K_c) >= q.k for every member k (raw and normalised
    q), equality for single-member clusters, and Eq. (1) equals the
    two-product form q+.Kmax + q-.Kmin."""
    cfg = synth.CONFIGS[1]
    Q, K, _ = synth.make_layer(cfg, heads=[0])
    p = orc.Params.from_layer_config(cfg)
    kc = orc.cluster_k_multistage(K[0], p)
    st = orc.key_stats(K[0], kc)
    nk = int(kc.n_k[0])
    X = synth.bf16_bits_to_f32(K[0, 0]).astype(np.float64)
    inv, xh = orc.qnorm(Q[0, 0][:200])
    for qs in (synth.bf16_bits_to_f32(Q[0, 0][:200]), xh):
        S = orc.quest(qs, st.kmax[0, :nk], st.kmin[0, :nk], st.counts[0, :nk])
        dots = qs.astype(np.float64) @ X.T
        for c in range(nk):
            m = kc.labels[0] == c
            if not m.any():
                assert np.isneginf(S[:, c]).all()
                continue
            mx = dots[:, m].max(1)
            assert (S[:, c] >= mx - 1e-4 * (np.abs(mx) + 1)).all()
        q = qs.astype(np.float64)
        two = np.maximum(q, 0) @ st.kmax[0, :nk].T.astype(np.float64) + \
            np.minimum(q, 0) @ st.kmin[0, :nk].T.astype(np.float64)
        ne = st.counts[0, :nk] > 0
        assert np.allclose(S[:, ne], two[:, ne], rtol=1e-5, atol=1e-4)
    # single-member cluster: the bound is attained
    k1 = X[:1].astype(np.float32)
    q1 = synth.bf16_bits_to_f32(Q[0, 0][:50])
    S1 = orc.quest(q1, k1, k1, np.array([1], np.int32))
    assert np.allclose(S1[:, 0], q1.astype(np.float64) @ k1[0].astype(np.float64), rtol=1e-5, atol=1e-5)


def test_mean_scores_hand_example():
    """The "w/o Quest" ablation (Sec. 4.4, Table 4): the score of a key cluster
    is q . mu with mu its centre; worked by hand in binary fractions (exact in
    fp32): q = [1, -2, 0.5], mu = [0.5, 0.25, -1] -> 0.5 - 0.5 - 0.5 = -0.5;
    an empty cluster scores -inf."""
    q = np.array([[1.0, -2.0, 0.5]], np.float32)
    mu = np.array([[0.5, 0.25, -1.0], [3.0, 3.0, 3.0]], np.float32)
    S = orc.mean_scores(q, mu, np.array([4, 0], np.int32))
    assert S[0, 0] == -0.5 and np.isneginf(S[0, 1])


def test_mean_scores_below_quest_and_equal_for_single_members():
    """mu_d lies between the members' min and max in every dimension, so
    q_d mu_d <= max(q_d Kmax_d, q_d Kmin_d) and the mean score never exceeds
    Eq. (1) (up to the rounding of the fp32 mean); a single-member cluster has
    mu = Kmax = Kmin, where the two scores are the same fp32 sum."""
    cfg = synth.CONFIGS[1]
    Q, K, _ = synth.make_layer(cfg, heads=[0])
    p = orc.Params.from_layer_config(cfg)
    kc = orc.cluster_k_multistage(K[0], p)
    st = orc.key_stats(K[0], kc)
    nk = int(kc.n_k[0])
    _, qh = orc.qnorm(Q[0, 0][:300])
    cnt = st.counts[0, :nk]
    Sq = orc.quest(qh, st.kmax[0, :nk], st.kmin[0, :nk], cnt)
    Sm = orc.mean_scores(qh, kc.C[0, :nk], cnt)
    ne = cnt > 0
    assert np.isneginf(Sm[:, ~ne]).all() and np.isfinite(Sm[:, ne]).all()
    scale = np.abs(qh).astype(np.float64) @ np.maximum(np.abs(st.kmax[0, :nk]), np.abs(st.kmin[0, :nk])).T
    assert (Sm[:, ne] <= Sq[:, ne] + 1e-6 * scale[:, ne]).all()
    # scores differ where clusters have several members
    assert (Sm[:, cnt > 1] < Sq[:, cnt > 1]).mean() > 0.9
    X = synth.bf16_bits_to_f32(K[0, 0][:40])
    one = np.ones(40, np.int32)
    assert np.array_equal(orc.mean_scores(qh, X, one), orc.quest(qh, X, X, one))


def _comp_case(seed, L=240, d=8, nk=12, dup=False):
    """A small head with random bf16 Q, K, V, random key clusters (or clusters
    of identical members when dup), one query cluster selecting 3 of them."""
    rng = np.random.default_rng(seed)
    labels_k = rng.integers(0, nk, L).astype(np.int32)
    labels_k[:nk] = np.arange(nk)  # every cluster non-empty
    if dup:
        proto_k = rng.normal(size=(nk, d)) * 0.8
        proto_v = rng.normal(size=(nk, d))
        Kf, Vf = proto_k[labels_k], proto_v[labels_k]
    else:
        Kf, Vf = rng.normal(size=(L, d)) * 0.8, rng.normal(size=(L, d))
    Qf = rng.normal(size=(L, d))
    Q16, K16, V16 = (synth.f32_to_bf16_bits(x.astype(np.float32)) for x in (Qf, Kf, Vf))
    sel = np.array([[1, 4, 7]], np.int32)
    return Q16, K16, V16, labels_k, sel


def test_compensation_error_identity():
    """ClusterAttention Sec. 1.2 Eq. (5): with w the dense softmax weights,
    w_bar_c the mean weight of cluster c, w_hat_c = exp(s(k_bar_c)) / Z the
    centroid's weight, delta_c = w_bar_c - w_hat_c, Cov_c the weight-value
    covariance of c and d_hat the compensated partition sum (relative to Z),
    o - o_hat = (1 / d_hat) sum_c |c| (delta_c (v_bar_c - o) + Cov_c) over
    the unselected clusters, exactly (here to fp64 rounding).  k_bar may be
    any point; v_bar must be the member mean."""
    Q16, K16, V16, labels_k, sel = _comp_case(3)
    L, d = K16.shape
    nk = 12
    Kf, Vf, Qf = (synth.bf16_bits_to_f32(x).astype(np.float64) for x in (K16, V16, Q16))
    cnt = np.bincount(labels_k, minlength=nk).astype(np.int32)
    vbar = np.stack([Vf[labels_k == c].mean(0) for c in range(nk)])
    kbar = np.stack([Kf[labels_k == c].mean(0) for c in range(nk)]) + 0.05  # any point will do
    rows = np.arange(0, L, 17)
    lq = np.zeros(L, np.int32)
    o = orc.attention_rows(Q16, K16, V16, lq, labels_k, None, True, rows)
    oh = orc.attention_rows_comp(Q16, K16, V16, lq, labels_k, sel, False, rows, nk, cnt, kbar, vbar)
    sc = 1.0 / np.sqrt(d)
    excl = [c for c in range(nk) if c not in sel[0]]
    for r, i in enumerate(rows):
        s = Kf @ Qf[i] * sc
        Z = np.exp(s).sum()
        w = np.exp(s) / Z
        dhat = w[np.isin(labels_k, sel[0])].sum()
        rhs = np.zeros(d)
        for c in excl:
            m = labels_k == c
            wb = w[m].mean()
            wh = np.exp(kbar[c] @ Qf[i] * sc) / Z
            dhat += cnt[c] * wh
            cov = ((w[m] - wb)[:, None] * (Vf[m] - vbar[c])).mean(0)
            rhs += cnt[c] * ((wb - wh) * (vbar[c] - o[r]) + cov)
        rhs /= dhat
        assert np.allclose(o[r] - oh[r], rhs, rtol=0, atol=1e-12), (i, np.abs(o[r] - oh[r] - rhs).max())
    # the unselected mass is not negligible here: compensation changes the output
    osel = orc.attention_rows(Q16, K16, V16, lq, labels_k, sel, False, rows)
    assert np.abs(osel - oh).max() > 1e-3


def test_compensation_exact_for_identical_members_and_all_selected():
    """Clusters of identical members: delta_c = 0 and Cov_c = 0, so the
    compensated output equals dense attention; with every cluster selected
    there is nothing to compensate."""
    Q16, K16, V16, labels_k, sel = _comp_case(5, dup=True)
    L, d = K16.shape
    nk = 12
    km, cnt = orc.cluster_means(K16, labels_k, nk)
    vm, _ = orc.cluster_means(V16, labels_k, nk)
    rows = np.arange(0, L, 11)
    lq = np.zeros(L, np.int32)
    o = orc.attention_rows(Q16, K16, V16, lq, labels_k, None, True, rows)
    oh = orc.attention_rows_comp(Q16, K16, V16, lq, labels_k, sel, False, rows, nk, cnt, km, vm)
    assert np.allclose(oh, o, rtol=0, atol=1e-12)
    Q16, K16, V16, labels_k, _ = _comp_case(6)
    km, cnt = orc.cluster_means(K16, labels_k, nk)
    vm, _ = orc.cluster_means(V16, labels_k, nk)
    every = np.arange(nk, dtype=np.int32)[None]
    o = orc.attention_rows(Q16, K16, V16, lq, labels_k, every, False, rows)
    oh = orc.attention_rows_comp(Q16, K16, V16, lq, labels_k, every, False, rows, nk, cnt, km, vm)
    assert np.array_equal(o, oh)


def test_compensated_layer_is_closer_to_dense():
    """Layer level (Params.compensate): the unselected key clusters enter as
    member-mean pseudo-tokens.  On the tiny layer, whose key clusters are tight
    mixture components, the compensated output lies closer to dense attention
    than the plain sparse one for most rows, and far closer on average."""
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg, heads=[0])
    B, H, L, d = Q.shape
    f = lambda x: x.reshape(B * H, L, d)  # noqa: E731
    p = orc.Params.from_layer_config(cfg)
    rows = np.arange(0, L, 29)
    plain = orc.layer(f(Q), f(K), f(V), p, rows=rows)
    p.compensate = 1
    comp = orc.layer(f(Q), f(K), f(V), p, rows=rows)
    assert not plain.kc.F[0]
    dense = orc.attention_rows(f(Q)[0], f(K)[0], f(V)[0], plain.labels_q[0], plain.kc.labels[0], None, True, rows)
    e_plain = np.linalg.norm(plain.O[0] - dense, axis=1)
    e_comp = np.linalg.norm(comp.O[0] - dense, axis=1)
    assert (e_comp < e_plain).mean() > 0.8 and e_comp.mean() < 0.5 * e_plain.mean()


def test_cluster_means_are_member_order_fp32_sums():
    """or_cluster_means follows the Lloyd update's rule (fp32 sums in ascending
    token order, then one division); a consistency check of that rule, not a
    pin: counts, the order-defined fp32 values, empty clusters 0."""
    rng = np.random.default_rng(2)
    X16 = synth.f32_to_bf16_bits(rng.normal(size=(500, 16)).astype(np.float32))
    lab = rng.integers(0, 9, 500).astype(np.int32)
    lab[lab == 4] = 5  # cluster 4 empty
    mean, cnt = orc.cluster_means(X16, lab, 9)
    Xf = synth.bf16_bits_to_f32(X16)
    for c in range(9):
        acc = np.zeros(16, np.float32)
        for j in np.nonzero(lab == c)[0]:
            acc = (acc + Xf[j]).astype(np.float32)
        n = int((lab == c).sum())
        assert cnt[c] == n
        want = (acc / np.float32(n)).astype(np.float32) if n else np.zeros(16, np.float32)
        assert np.array_equal(mean[c], want)


def test_tail_merge_worked_example():
    """The worked example of iCATS's tail merging (tests/golden/tail_merge_example.json):
    query clusters #12 and #45 (210 and 180 tokens) attend to the same key
    clusters and merge into #12 (390); #3 (300 tokens, tail 44) and #18 (170,
    tail 42) are each other's nearest masks and 44 + 42 <= 128, so #18's last
    42 tokens move to #3, whose mask becomes the union."""
    g = _golden("tail_merge_example.json")
    b = g["b"]
    sizes = {3: 300, 12: 210, 18: 170, 45: 180}
    nk = 8
    masks = np.zeros((46, nk), bool)
    masks[12, [0, 1]] = masks[45, [0, 1]] = True
    masks[3, [2, 3, 4]] = True
    masks[18, [2, 3, 5]] = True
    rng = np.random.default_rng(4)
    labels = np.concatenate([np.full(n, c, np.int32) for c, n in sizes.items()])
    rng.shuffle(labels)
    owner, new_masks, groups, pairs = orc.tail_merge(labels, masks, b)
    s1 = g["stage1"]
    assert len(groups[s1["merged_into"]]) == s1["merged_size"] == sum(s1["sizes"])
    s2 = g["stage2"]
    assert [sizes[c] % b for c in s2["clusters"]] == s2["tails"] and sum(s2["tails"]) == s2["tail_sum"] <= b
    assert pairs == [(s2["tokens_moved_to"], s2["tokens_moved_from"], s2["moved"])]
    last = np.nonzero(labels == s2["tokens_moved_from"])[0][-s2["moved"]:]
    assert (owner[last] == s2["tokens_moved_to"]).all()
    assert len(groups[3]) == 300 + 42 and len(groups[18]) == 128
    assert np.array_equal(new_masks[3], masks[3] | masks[18])
    # the 390-token group keeps its tail: its nearest mask (#3) pairs with #18
    assert np.array_equal(new_masks[12], masks[12])


def test_tail_merge_invariants():
    """Every token keeps exactly one owner; tiles never increase; a token's key
    set after merging contains its own cluster's; stage 1 changes no token's
    key set; paired tails fit one tile and leave the donor aligned."""
    rng = np.random.default_rng(12)
    b, Cq, nk = 128, 24, 40
    base = rng.random((8, nk)) < 0.2
    masks = base[rng.integers(0, 8, Cq)] | (rng.random((Cq, nk)) < 0.03)
    masks[5] = masks[2]
    masks[9] = masks[2]
    labels = rng.integers(0, Cq, 4000).astype(np.int32)
    owner, new_masks, groups, pairs = orc.tail_merge(labels, masks, b)
    assert (owner >= 0).all() and sorted(np.concatenate([np.asarray(t) for t in groups.values()])) == list(range(4000))
    sizes = np.bincount(labels, minlength=Cq)
    before = int(np.sum((sizes + b - 1) // b))
    after = int(sum((len(t) + b - 1) // b for t in groups.values()))
    assert after <= before
    moved = set()
    for i, j, n in pairs:
        assert 0 < n < b and (len(groups[j]) % b) == 0
        moved.update(np.nonzero(owner == i)[0].tolist())
    for t in range(4000):
        mine = masks[labels[t]]
        assert (new_masks[owner[t]] >= mine).all()
        if owner[t] not in [i for i, _, _ in pairs]:
            assert np.array_equal(new_masks[owner[t]], mine)
    # clusters 5 and 9 share cluster 2's mask: stage 1 folds them into 2
    assert 2 in groups and 5 not in groups and 9 not in groups


def test_topk_bruteforce_with_ties_and_empties():
    rng = np.random.default_rng(9)
    S = rng.integers(0, 6, size=(20, 30)).astype(np.float32)
    S[:, 7] = -np.inf
    k = 9
    sel = orc.topk(S, k)
    for a in range(20):
        order = sorted(range(30), key=lambda c: (-S[a, c], c))[:k]
        assert sel[a].tolist() == sorted(order)
        assert 7 not in sel[a]


def test_topk_count_rule():
    assert orc.topk_count(8, 100, 100) == 8
    assert orc.topk_count(-100, 500, 500) == 50
    assert orc.topk_count(-100, 501, 501) == 51      # ceil
    assert orc.topk_count(-50, 10, 10) == 1
    assert orc.topk_count(64, 100, 20) == 20          # clamp to non-empty
    assert orc.topk_count(-1, 3, 3) == 1              # at least one


# ----------------------------------------------------------------- attention

def test_attention_hand_example():
    g = _golden("quest_attention_hand.json")["attention"]
    Q = bf([g["q"]])
    K = bf(g["keys"])
    V = bf(g["values"])
    o = orc.attention_rows(Q, K, V, np.zeros(1, np.int32), np.zeros(2, np.int32), None, True,
                           [0], scale=g["scale"])
    assert np.allclose(o[0], g["out"], atol=1e-15)


def test_dense_attention_equals_torch_sdpa():
    import torch
    rng = np.random.default_rng(10)
    L, d = 300, 64
    Q, K, V = (bf(rng.standard_normal((L, d))) for _ in range(3))
    o = orc.attention_rows(Q, K, V, np.zeros(L, np.int32), np.zeros(L, np.int32), None, True,
                           np.arange(L))
    t = [torch.from_numpy(synth.bf16_bits_to_f32(x).astype(np.float64))[None, None] for x in (Q, K, V)]
    ref = torch.nn.functional.scaled_dot_product_attention(*t)[0, 0].numpy()
    assert np.abs(o - ref).max() < 1e-12


def test_all_selected_equals_dense_and_error_split():
    """Check (a): selecting every non-empty key cluster gives dense attention.
    Check (d): o - o_S = (1 - w_S)(o_Sbar - o_S) (ClusterAttention Sec. 1.2,
    Eq. (3)-(4)) with S the keys of the selected clusters."""
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg, heads=[0])
    Q, K, V = Q[0, 0], K[0, 0], V[0, 0]
    p = orc.Params.from_layer_config(cfg)
    r = orc.layer(Q[None], K[None], V[None], p, attention=False)
    nk = int(r.kc.n_k[0])
    lq, lk = r.labels_q[0], r.kc.labels[0]
    rows = np.arange(0, cfg.L, 97)
    allsel = np.tile(np.arange(nk, dtype=np.int32), (cfg.Cq, 1))
    o_all = orc.attention_rows(Q, K, V, lq, lk, allsel, False, rows)
    o_dense = orc.attention_rows(Q, K, V, lq, lk, None, True, rows)
    assert np.abs(o_all - o_dense).max() < 1e-12
    sel = r.sel[0]
    o_S = orc.attention_rows(Q, K, V, lq, lk, sel, False, rows)
    Vf = synth.bf16_bits_to_f32(V).astype(np.float64)
    for n, i in enumerate(rows):
        w = orc.dense_weights(Q[i], K)
        inS = np.isin(lk, sel[lq[i]])
        wS = w[inS].sum()
        comp = [c for c in range(nk) if c not in set(sel[lq[i]].tolist())]
        o_Sbar = orc.attention_rows(Q, K, V, lq, lk, np.array([comp] * cfg.Cq, np.int32), False,
                                    [i])[0] if comp else np.zeros(cfg.d)
        lhs = o_dense[n] - o_S[n]
        rhs = (1 - wS) * (o_Sbar - o_S[n])
        assert np.abs(lhs - rhs).max() < 1e-5
        # and o itself is the weighted combination (Eq. (3))
        assert np.abs(o_dense[n] - (w[:, None] * Vf).sum(0)).max() < 1e-10
