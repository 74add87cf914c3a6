"""Pins of the oracle's warm-started steps (AdaCluster Sec. 3.2.2 "Efficient
initialization": the cluster count of the first denoising step is kept and the
previous centres start the Lloyd iterations of the next step).

or_cluster_k_warm and the init branch of or_cluster_q are checked against
things other than themselves: scikit-learn's Lloyd k-means started from the
same centres, a Lloyd fixed point (which a warm step must leave alone), and
the bookkeeping a warm step must not touch (dense heads, centre slots past
n_k)."""
import numpy as np

from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth


def _mixture(rng, n, d, centres, spread):
    comp = rng.integers(0, centres.shape[0], n)
    return (centres[comp] + spread * rng.standard_normal((n, d))).astype(np.float32)


def _bf16(x):
    return synth.f32_to_bf16_bits(x)


def _kc(labels, C, n_k, F):
    BH, L = labels.shape
    return orc.KClusters(labels, C, n_k, F, 0.0, np.zeros(BH, np.int32), np.full((BH, L), -1, np.int32),
                         np.zeros((BH, L), np.float32))


def test_warm_keys_match_sklearn_lloyd_per_head():
    """Each head: T Lloyd iterations from its own first n_k centres, as scikit-learn's
    Lloyd k-means started there; other heads' counts and strides must not leak in."""
    from sklearn.cluster import KMeans
    rng = np.random.default_rng(21)
    BH, L, d, ccap, T = 3, 900, 8, 20, 2
    n_k = np.array([5, 9, 14], np.int32)
    K16 = np.empty((BH, L, d), np.uint16)
    C = rng.standard_normal((BH, ccap, d)).astype(np.float32) * 50  # slots past n_k: junk
    for h in range(BH):
        centres = rng.standard_normal((n_k[h], d)) * 8
        K16[h] = _bf16(_mixture(rng, L, d, centres, 1.0))
        C[h, :n_k[h]] = (centres + 0.5 * rng.standard_normal(centres.shape)).astype(np.float32)
    p = orc.Params(Cq=4, m0=4, n_max=ccap - 4, tau_mode=orc.TAU_ABSOLUTE, tau_value=1.0, topk=1, iters_warm=T)
    prev = _kc(np.zeros((BH, L), np.int32), C.copy(), n_k.copy(), np.zeros(BH, np.uint8))
    out = orc.cluster_k_warm(K16, p, prev)
    for h in range(BH):
        X = synth.bf16_bits_to_f32(K16[h]).astype(np.float64)
        km = KMeans(n_clusters=int(n_k[h]), init=C[h, :n_k[h]].astype(np.float64), n_init=1, max_iter=T,
                    tol=0.0, algorithm="lloyd").fit(X)
        np.testing.assert_array_equal(out.labels[h], km.labels_)
        assert np.allclose(out.C[h, :n_k[h]], km.cluster_centers_, rtol=1e-5, atol=1e-5)
        # the slots past n_k are not the head's centres: untouched, bit for bit
        np.testing.assert_array_equal(out.C[h, n_k[h]:], C[h, n_k[h]:])
    np.testing.assert_array_equal(out.n_k, n_k)


def test_warm_keys_leave_a_lloyd_fixed_point_unchanged():
    """Centres that are already the member means of a partition that assigns to
    itself are a fixed point of Lloyd's map: a warm step changes nothing."""
    rng = np.random.default_rng(22)
    L, d, m = 1200, 16, 12
    centres = rng.standard_normal((m, d)) * 10
    X16 = _bf16(_mixture(rng, L, d, centres, 0.5))
    X = synth.bf16_bits_to_f32(X16)
    lab, _, C = orc.kmeans(X, X[orc.seed_pick(3, 0, 0, L, m)], 60)  # converged
    C2, _ = orc.update(X, lab, C)
    assert np.array_equal(C2, C), "not converged: pick more iterations"
    ccap = m + 3
    Cfull = np.zeros((1, ccap, d), np.float32)
    Cfull[0, :m] = C
    p = orc.Params(Cq=4, m0=3, n_max=m, tau_mode=orc.TAU_ABSOLUTE, tau_value=1.0, topk=1, iters_warm=2)
    out = orc.cluster_k_warm(X16[None], p, _kc(np.zeros((1, L), np.int32), Cfull, np.array([m], np.int32),
                                               np.zeros(1, np.uint8)))
    np.testing.assert_array_equal(out.labels[0], lab)
    np.testing.assert_array_equal(out.C[0], Cfull[0])


def test_warm_keys_skip_dense_heads_bit_for_bit():
    """A head whose dense flag F is set keeps its labels and centres untouched."""
    rng = np.random.default_rng(23)
    BH, L, d, ccap = 2, 400, 8, 10
    K16 = _bf16(rng.standard_normal((BH, L, d)).astype(np.float32))
    C = rng.standard_normal((BH, ccap, d)).astype(np.float32)
    labels = rng.integers(0, 6, (BH, L)).astype(np.int32)
    p = orc.Params(Cq=4, m0=4, n_max=6, tau_mode=orc.TAU_ABSOLUTE, tau_value=1.0, topk=1, iters_warm=2)
    out = orc.cluster_k_warm(K16, p, _kc(labels.copy(), C.copy(), np.array([6, 6], np.int32),
                                         np.array([1, 0], np.uint8)))
    np.testing.assert_array_equal(out.labels[0], labels[0])
    np.testing.assert_array_equal(out.C[0], C[0])
    assert not np.array_equal(out.C[1, :6], C[1, :6])  # the sparse head did run


def test_warm_queries_from_init_match_sklearn_on_normalised_queries():
    """or_cluster_q with init: Lloyd from the given centres on the L2-normalised
    queries (centres stay plain means), as scikit-learn does on the same unit
    vectors; with zero iterations, the labels are the nearest given centres and
    the centres are returned unchanged."""
    from sklearn.cluster import KMeans
    cfg = synth.CONFIGS[1]
    Q16, _, _ = synth.make_layer(cfg)
    Q16 = Q16.reshape(-1, cfg.L, cfg.d)
    p = orc.Params.from_layer_config(cfg, seed=99)
    lab0, C0, _ = orc.cluster_q(Q16, p)  # a previous step's centres
    rng = np.random.default_rng(24)
    init = (C0 + 0.01 * rng.standard_normal(C0.shape)).astype(np.float32)
    lab, C, cnt = orc.cluster_q(Q16, p, init=init, iters=2)
    for h in range(Q16.shape[0]):
        _, xh = orc.qnorm(Q16[h])
        km = KMeans(n_clusters=cfg.Cq, init=init[h].astype(np.float64), n_init=1, max_iter=2, tol=0.0,
                    algorithm="lloyd").fit(xh.astype(np.float64))
        D = ((xh[:, None, :].astype(np.float64) - km.cluster_centers_[None]) ** 2).sum(-1)
        srt = np.sort(D, axis=1)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-6 * np.maximum(srt[:, 0], 1e-12)
        assert clear.mean() > 0.99
        np.testing.assert_array_equal(lab[h][clear], km.labels_[clear])
        assert np.allclose(C[h], km.cluster_centers_, rtol=1e-5, atol=1e-6)
        np.testing.assert_array_equal(cnt[h], np.bincount(lab[h], minlength=cfg.Cq))
    lab_z, C_z, _ = orc.cluster_q(Q16, p, init=init, iters=0)
    np.testing.assert_array_equal(C_z, init)
    for h in range(Q16.shape[0]):
        _, xh = orc.qnorm(Q16[h])
        D = ((xh[:, None, :].astype(np.float64) - init[h][None].astype(np.float64)) ** 2).sum(-1)
        srt = np.sort(D, axis=1)
        clear = (srt[:, 1] - srt[:, 0]) > 1e-6 * np.maximum(srt[:, 0], 1e-12)
        np.testing.assert_array_equal(lab_z[h][clear], D.argmin(1)[clear])


def test_head_subset_uses_the_layer_seeds():
    """A head run on its own with unit0 = its index (and the layer's tau given as
    an absolute threshold) reproduces that head of the whole-layer run."""
    cfg = synth.CONFIGS[1]
    Q16, K16, _ = synth.make_layer(cfg)
    Q16, K16 = Q16.reshape(-1, cfg.L, cfg.d), K16.reshape(-1, cfg.L, cfg.d)
    p = orc.Params.from_layer_config(cfg, seed=5)
    lab_q, C_q, _ = orc.cluster_q(Q16, p)
    kc = orc.cluster_k_multistage(K16, p)
    import dataclasses
    ph = dataclasses.replace(p, tau_mode=orc.TAU_ABSOLUTE, tau_value=kc.tau, unit0=1)
    lab_q1, C_q1, _ = orc.cluster_q(Q16[1:2], ph)
    kc1 = orc.cluster_k_multistage(K16[1:2], ph)
    np.testing.assert_array_equal(lab_q1[0], lab_q[1])
    np.testing.assert_array_equal(C_q1[0], C_q[1])
    np.testing.assert_array_equal(kc1.labels[0], kc.labels[1])
    np.testing.assert_array_equal(kc1.C[0], kc.C[1])
    assert kc1.n_k[0] == kc.n_k[1] and kc1.stages[0] == kc.stages[1]
    # and unit0 = 0 on head 1 draws other seeds (the pin has teeth)
    lab_q0, _, _ = orc.cluster_q(Q16[1:2], dataclasses.replace(ph, unit0=0))
    assert not np.array_equal(lab_q0[0], lab_q[1])
