"""CPU oracle of the cluster-routed sparse attention layer (Python side).

TEST INFRASTRUCTURE ONLY: tests/, __graft_entry__.smoke() and the cpu_baseline /
reference legs of bench.py may import this module; the CUDA product never does.
It shares no code with the product; the only common module is the seeded input
generator (cluster_routed_sparse_b200.synth), which holds none of the method's
arithmetic.

The arithmetic lives in ac_oracle.c (plain C, compiled here with gcc,
-ffp-contract=off); this file marshals numpy arrays and strings the steps
together in the order of Algorithm 3 of "AdaCluster: Adaptive Query-Key
Clustering for Sparse Attention in Video Generation":
  line 3   A_q, C_q <- KMeans(Normalize(Q))
  line 4   A_k, C_k, F <- MultiStageClustering(K, tau, N_max)   (Algorithm 1)
  line 8   S <- TensorQuest(...)                                (Eq. (1))
  line 9   Index <- argtopk(S, topk)
  line 11  AttnOut <- Attention(Q, K*, V*)   (line 6: dense when F is set)
"""
from __future__ import annotations

import ctypes
import dataclasses
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ac_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")

TAU_ABSOLUTE, TAU_MEAN_FACTOR, TAU_PERCENTILE = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile ac_oracle.c into liboracle.so next to it (gcc, OpenMP)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        cmd = ["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-fPIC",
               "-shared", "-Wall", "-o", _LIB + ".tmp", _SRC, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(_LIB + ".tmp", _LIB)
    return _LIB


class _Cfg(ctypes.Structure):
    _fields_ = [("Cq", ctypes.c_int), ("m0", ctypes.c_int), ("n_max", ctypes.c_int),
                ("tau_mode", ctypes.c_int), ("tau_value", ctypes.c_float),
                ("topk", ctypes.c_int), ("iters_q", ctypes.c_int), ("iters_k", ctypes.c_int),
                ("iters_warm", ctypes.c_int), ("stage_rule", ctypes.c_int),
                ("seed", ctypes.c_uint64), ("unit0", ctypes.c_int64)]


_lib = None


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        _lib.or_rand.restype = ctypes.c_uint64
        _lib.or_rand.argtypes = [ctypes.c_uint64, ctypes.c_int64, ctypes.c_int32, ctypes.c_int64]
        _lib.or_tau.restype = ctypes.c_float
        _lib.or_tau.argtypes = [ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_float]
        _lib.or_objective.restype = ctypes.c_double
        _lib.or_topk_count.restype = ctypes.c_int32
        _lib.or_topk_count.argtypes = [ctypes.c_int32] * 3
        _lib.or_stage_clusters.restype = ctypes.c_int32
        _lib.or_stage_clusters.argtypes = [ctypes.c_int32, ctypes.c_int64, ctypes.c_int64, ctypes.c_int,
                                           ctypes.c_int]
        _lib.or_cluster_k_multistage.restype = ctypes.c_int
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p) if a is not None else None


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


@dataclasses.dataclass
class Params:
    """Method hyper-parameters (field meanings as in ac_oracle.c's or_cfg)."""
    Cq: int
    m0: int
    n_max: int
    tau_mode: int
    tau_value: float
    topk: int
    iters_q: int = 10
    iters_k: int = 10
    iters_warm: int = 2
    seed: int = 1234
    stage_rule: int = 0
    score_mode: int = 0   # 0: Eq. (1) bound; 1: mean-based scores (the "w/o Quest" ablation)
    tail_merge: int = 0   # 0: off; 1: stage 1 of tail_merge (lossless); 2: both stages
    compensate: int = 0   # 1: unselected clusters enter as centroid pseudo-tokens (attention_rows_comp)
    unit0: int = 0        # (batch, head) index of the first unit of a call (the seeds of a head subset)

    @property
    def ccap(self) -> int:
        return self.n_max + self.m0

    def c(self) -> _Cfg:
        return _Cfg(self.Cq, self.m0, self.n_max, self.tau_mode, float(self.tau_value),
                    self.topk, self.iters_q, self.iters_k, self.iters_warm, self.stage_rule,
                    ctypes.c_uint64(self.seed & (2**64 - 1)), ctypes.c_int64(self.unit0))

    @staticmethod
    def from_layer_config(cfg, seed: int = 1234) -> "Params":
        return Params(cfg.Cq, cfg.m0, cfg.n_max, cfg.tau_mode, cfg.tau_value, cfg.topk,
                      cfg.iters_q, cfg.iters_k, cfg.iters_warm, seed, cfg.stage_rule)


# ---------------------------------------------------------------- single steps

def rand(seed: int, bh: int, tag: int, i: int) -> int:
    return int(lib().or_rand(seed, bh, tag, i))


def seed_pick(seed: int, bh: int, tag: int, n: int, m: int) -> np.ndarray:
    pos = np.empty(m, np.int64)
    lib().or_seed_pick(ctypes.c_uint64(seed), ctypes.c_int64(bh), ctypes.c_int32(tag),
                       ctypes.c_int64(n), ctypes.c_int32(m), _p(pos))
    return pos


def qnorm(Q16: np.ndarray):
    """(inv [rows], xhat [rows, d] fp32) for bf16 rows Q16 [..., d]."""
    Q16 = _c(Q16, np.uint16)
    d = Q16.shape[-1]
    rows = Q16.size // d
    inv = np.empty(rows, np.float32)
    xh = np.empty((rows, d), np.float32)
    lib().or_qnorm(_p(Q16), ctypes.c_int64(rows), ctypes.c_int(d), _p(inv), _p(xh))
    return inv, xh


def assign(X: np.ndarray, C: np.ndarray):
    X = _c(X, np.float32)
    C = _c(C, np.float32)
    n, d = X.shape
    lab = np.empty(n, np.int32)
    dm = np.empty(n, np.float32)
    lib().or_assign(_p(X), ctypes.c_int64(n), ctypes.c_int(d), _p(C), ctypes.c_int(C.shape[0]),
                    _p(lab), _p(dm))
    return lab, dm


def update(X: np.ndarray, labels: np.ndarray, C_prev: np.ndarray):
    X = _c(X, np.float32)
    C = _c(C_prev, np.float32).copy()
    n, d = X.shape
    cnt = np.empty(C.shape[0], np.int32)
    lib().or_update(_p(X), ctypes.c_int64(n), ctypes.c_int(d), _p(_c(labels, np.int32)),
                    ctypes.c_int(C.shape[0]), _p(C), _p(cnt))
    return C, cnt


def objective(X, C, labels) -> float:
    X = _c(X, np.float32)
    return float(lib().or_objective(_p(X), ctypes.c_int64(X.shape[0]), ctypes.c_int(X.shape[1]),
                                    _p(_c(C, np.float32)), _p(_c(labels, np.int32))))


def kmeans(X: np.ndarray, C_init: np.ndarray, T: int, trace: bool = False):
    """T Lloyd iterations then a final assignment: (labels, dmin, C[, J trace])."""
    X = _c(X, np.float32)
    C = _c(C_init, np.float32).copy()
    n, d = X.shape
    lab = np.empty(n, np.int32)
    dm = np.empty(n, np.float32)
    jt = np.empty(2 * T + 1, np.float64) if trace else None
    lib().or_kmeans(_p(X), ctypes.c_int64(n), ctypes.c_int(d), _p(C), ctypes.c_int(C.shape[0]),
                    ctypes.c_int(T), _p(lab), _p(dm), _p(jt))
    return (lab, dm, C, jt) if trace else (lab, dm, C)


def tau(dist: np.ndarray, mode: int, value: float) -> float:
    dist = _c(dist, np.float32)
    return float(lib().or_tau(_p(dist), ctypes.c_int64(dist.size), ctypes.c_int(mode),
                              ctypes.c_float(value)))


def stage_clusters(m0: int, nU: int, L: int, t: int, rule: int = 0) -> int:
    return int(lib().or_stage_clusters(m0, nU, L, t, rule))


def topk_count(topk: int, nk: int, nonempty: int) -> int:
    return int(lib().or_topk_count(topk, nk, nonempty))


# ---------------------------------------------------------------- layer steps

def cluster_q(Q16: np.ndarray, p: Params, init=None, iters=None):
    """Angular k-means of the queries of every head.  Q16: [BH, L, d] bf16 bits.
    Returns (labels [BH, L], centres [BH, Cq, d], counts [BH, Cq])."""
    Q16 = _c(Q16, np.uint16)
    BH, L, d = Q16.shape
    lab = np.empty((BH, L), np.int32)
    C = np.empty((BH, p.Cq, d), np.float32)
    cnt = np.empty((BH, p.Cq), np.int32)
    cfg = p.c()
    T = p.iters_q if iters is None else iters
    lib().or_cluster_q(_p(Q16), ctypes.c_int(BH), ctypes.c_int(L), ctypes.c_int(d),
                       ctypes.byref(cfg), _p(None if init is None else _c(init, np.float32)),
                       ctypes.c_int(T), _p(lab), _p(C), _p(cnt))
    return lab, C, cnt


@dataclasses.dataclass
class KClusters:
    labels: np.ndarray        # [BH, L] int32
    C: np.ndarray             # [BH, Ccap, d] fp32
    n_k: np.ndarray           # [BH] int32
    F: np.ndarray             # [BH] uint8
    tau: float
    stages: np.ndarray        # [BH] int32
    removed_stage: np.ndarray  # [BH, L] int32
    removed_dist: np.ndarray   # [BH, L] fp32


def cluster_k_multistage(K16: np.ndarray, p: Params) -> KClusters:
    """Algorithm 1 on every head; tau pooled over the heads of the call."""
    K16 = _c(K16, np.uint16)
    BH, L, d = K16.shape
    cc = p.ccap
    lab = np.empty((BH, L), np.int32)
    C = np.zeros((BH, cc, d), np.float32)
    nk = np.empty(BH, np.int32)
    F = np.empty(BH, np.uint8)
    st = np.empty(BH, np.int32)
    rs = np.empty((BH, L), np.int32)
    rd = np.zeros((BH, L), np.float32)
    t = ctypes.c_float(0)
    cfg = p.c()
    rc = lib().or_cluster_k_multistage(_p(K16), ctypes.c_int(BH), ctypes.c_int(L), ctypes.c_int(d),
                                       ctypes.byref(cfg), _p(lab), _p(C), _p(nk), _p(F),
                                       ctypes.byref(t), _p(st), _p(rs), _p(rd))
    if rc != 0:
        raise ValueError("invalid multi-stage parameters")
    return KClusters(lab, C, nk, F, float(t.value), st, rs, rd)


def cluster_k_warm(K16, p: Params, kc: KClusters, iters=None) -> KClusters:
    """Warm-started step: n_k kept, previous centres as init, dense heads skipped."""
    K16 = _c(K16, np.uint16)
    BH, L, d = K16.shape
    C = kc.C.copy()
    lab = kc.labels.copy()
    T = p.iters_warm if iters is None else iters
    lib().or_cluster_k_warm(_p(K16), ctypes.c_int(BH), ctypes.c_int(L), ctypes.c_int(d),
                            ctypes.c_int(C.shape[1]), _p(_c(kc.n_k, np.int32)),
                            _p(_c(kc.F, np.uint8)), ctypes.c_int(T), _p(C), _p(lab))
    return dataclasses.replace(kc, labels=lab, C=C)


@dataclasses.dataclass
class KStats:
    counts: np.ndarray   # [BH, Ccap] int32
    kmax: np.ndarray     # [BH, Ccap, d] fp32 (exact bf16 values)
    kmin: np.ndarray
    sse: np.ndarray      # [BH, Ccap]
    mse: np.ndarray      # [BH]
    comp: np.ndarray     # [BH]


def key_stats(K16, kc: KClusters) -> KStats:
    K16 = _c(K16, np.uint16)
    BH, L, d = K16.shape
    cc = kc.C.shape[1]
    cnt = np.empty((BH, cc), np.int32)
    mx = np.empty((BH, cc, d), np.float32)
    mn = np.empty((BH, cc, d), np.float32)
    se = np.empty((BH, cc), np.float32)
    mse = np.empty(BH, np.float32)
    comp = np.empty(BH, np.float32)
    lib().or_key_stats(_p(K16), ctypes.c_int(BH), ctypes.c_int(L), ctypes.c_int(d), ctypes.c_int(cc),
                       _p(_c(kc.n_k, np.int32)), _p(_c(kc.labels, np.int32)),
                       _p(_c(kc.C, np.float32)), _p(cnt), _p(mx), _p(mn), _p(se), _p(mse), _p(comp))
    return KStats(cnt, mx, mn, se, mse, comp)


def quest(qc: np.ndarray, kmax: np.ndarray, kmin: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Eq. (1) scores of one head: qc [nq, d], kmax/kmin [nk, d] -> S [nq, nk]."""
    qc = _c(qc, np.float32)
    nq, d = qc.shape
    nk = kmax.shape[0]
    S = np.empty((nq, nk), np.float32)
    lib().or_quest(_p(qc), ctypes.c_int(nq), ctypes.c_int(d), _p(_c(kmax, np.float32)),
                   _p(_c(kmin, np.float32)), _p(_c(counts, np.int32)), ctypes.c_int(nk), _p(S))
    return S


def mean_scores(qc: np.ndarray, cent: np.ndarray, counts: np.ndarray) -> np.ndarray:
    """Mean-based scores of one head (Sec. 4.4 Table 4 "w/o Quest"): qc [nq, d],
    key-cluster centres cent [nk, d] -> S [nq, nk]."""
    qc = _c(qc, np.float32)
    nq, d = qc.shape
    nk = cent.shape[0]
    S = np.empty((nq, nk), np.float32)
    lib().or_mean_scores(_p(qc), ctypes.c_int(nq), ctypes.c_int(d), _p(_c(cent, np.float32)),
                         _p(_c(counts, np.int32)), ctypes.c_int(nk), _p(S))
    return S


def topk(S: np.ndarray, k: int) -> np.ndarray:
    S = _c(S, np.float32)
    nq, nk = S.shape
    sel = np.empty((nq, k), np.int32)
    lib().or_topk(_p(S), ctypes.c_int(nq), ctypes.c_int(nk), ctypes.c_int32(k), _p(sel))
    return sel


def score_select(Cq: np.ndarray, st: KStats, n_k: np.ndarray, topk_param: int, score_mode: int = 0,
                 Ck: np.ndarray | None = None):
    """Per head: S = Eq.(1) (score_mode 0) or the mean-based scores against the
    key centres Ck [BH, Ccap, d] (score_mode 1) over the n_k clusters,
    k = topk_count, Sel [Cq, k].  Returns (list of S [Cq, n_k], list of Sel, k per head)."""
    Ss, sels, ks = [], [], []
    for h in range(Cq.shape[0]):
        nk = int(n_k[h])
        cnt = st.counts[h, :nk]
        if score_mode == 1:
            S = mean_scores(Cq[h], Ck[h, :nk], cnt)
        else:
            S = quest(Cq[h], st.kmax[h, :nk], st.kmin[h, :nk], cnt)
        k = topk_count(topk_param, nk, int((cnt > 0).sum()))
        Ss.append(S)
        sels.append(topk(S, k))
        ks.append(k)
    return Ss, sels, np.array(ks, np.int32)


def attention_rows(Q16h, K16h, V16h, labels_q, labels_k, sel, dense: bool, rows,
                   scale: float | None = None) -> np.ndarray:
    """Algorithm 3 lines 5-11 for the listed query rows of one head (fp64)."""
    Q16h = _c(Q16h, np.uint16)
    K16h = _c(K16h, np.uint16)
    L, d = K16h.shape          # keys of the head (queries are indexed by rows)
    rows = _c(rows, np.int64)
    out = np.empty((rows.size, d), np.float64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    if sel is None:
        sel = np.zeros((1, 1), np.int32)
        dense = True
    sel = _c(sel, np.int32)
    lib().or_attention_rows(_p(Q16h), _p(_c(K16h, np.uint16)), _p(_c(V16h, np.uint16)),
                            ctypes.c_int(L), ctypes.c_int(d), _p(_c(labels_q, np.int32)),
                            _p(_c(labels_k, np.int32)), _p(sel), ctypes.c_int32(sel.shape[1]),
                            ctypes.c_int(1 if dense else 0), ctypes.c_double(sc), _p(rows),
                            ctypes.c_int64(rows.size), _p(out))
    return out


def cluster_means(X16h: np.ndarray, labels: np.ndarray, nk: int):
    """Member means of the clusters c < nk of one head (fp32, ascending token
    order, as the Lloyd update) and their counts."""
    X16h = _c(X16h, np.uint16)
    L, d = X16h.shape
    mean = np.empty((max(nk, 1), d), np.float32)
    cnt = np.empty(max(nk, 1), np.int32)
    lib().or_cluster_means(_p(X16h), ctypes.c_int(L), ctypes.c_int(d), _p(_c(labels, np.int32)),
                           ctypes.c_int(nk), _p(mean), _p(cnt))
    return mean[:nk], cnt[:nk]


def attention_rows_comp(Q16h, K16h, V16h, labels_q, labels_k, sel, dense: bool, rows, nk: int,
                        counts, kbar, vbar, scale: float | None = None) -> np.ndarray:
    """attention_rows with the unselected clusters compensated by their centroids
    (ClusterAttention Sec. 1.2 Eq. (5)-(6)): kbar / vbar [nk, d] (fp64), counts [nk]."""
    Q16h = _c(Q16h, np.uint16)
    K16h = _c(K16h, np.uint16)
    L, d = K16h.shape
    rows = _c(rows, np.int64)
    out = np.empty((rows.size, d), np.float64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    if sel is None:
        sel = np.zeros((1, 1), np.int32)
        dense = True
    sel = _c(sel, np.int32)
    lib().or_attention_rows_comp(_p(Q16h), _p(K16h), _p(_c(V16h, np.uint16)), ctypes.c_int(L), ctypes.c_int(d),
                                 _p(_c(labels_q, np.int32)), _p(_c(labels_k, np.int32)), _p(sel),
                                 ctypes.c_int32(sel.shape[1]), ctypes.c_int(1 if dense else 0),
                                 ctypes.c_double(sc), _p(rows), ctypes.c_int64(rows.size), ctypes.c_int(nk),
                                 _p(_c(counts, np.int32)), _p(_c(kbar, np.float64)), _p(_c(vbar, np.float64)),
                                 _p(out))
    return out


def tail_merge(labels_q: np.ndarray, masks: np.ndarray, b: int = 128, stages: int = 2):
    """Two-stage tail merging of one head's query clusters (iCATS, "tail merging
    strategy" and its worked example), for a kernel that runs query clusters in
    b-row tiles.  labels_q [L]: query cluster of each token; masks [Cq, nk] bool:
    the key clusters each query cluster attends to.

    Stage 1 (lossless): query clusters with identical masks form one group,
    owned by its lowest-index member; a group's tokens are its members' tokens,
    member by member in cluster order, each in ascending token order.
    Stage 2 (tail remap): among the groups whose size has a tail
    t = size mod b > 0, each finds its nearest neighbour by the Hamming
    distance of the masks (ties to the lower index); two groups that are each
    other's nearest neighbour and whose tails fit one tile (t_i + t_j <= b)
    pair up: the higher-index group j hands its last t_j tokens to the
    lower-index group i, and i's mask becomes the union of both.
    Readings: the pages do not say which cluster of a pair absorbs the other's
    tail (their example is consistent with either); here the lower index does.

    stages = 1 skips stage 2.
    Returns (owner [L] int32: the group whose mask each token attends with,
    new_masks [Cq, nk] bool, groups {owner: token list in group order},
    pairs [(i, j, moved)])."""
    labels_q = np.asarray(labels_q)
    masks = np.asarray(masks, bool)
    Cq = masks.shape[0]
    members = [np.nonzero(labels_q == c)[0] for c in range(Cq)]
    # stage 1: identical masks
    rep = list(range(Cq))
    for c in range(Cq):
        if members[c].size == 0:
            continue
        for r in range(c):
            if members[r].size and rep[r] == r and np.array_equal(masks[r], masks[c]):
                rep[c] = r
                break
    groups = {}
    for c in range(Cq):
        if members[c].size:
            groups.setdefault(rep[c], []).extend(members[c].tolist())
    new_masks = masks.copy()
    # stage 2: mutual nearest neighbours among the groups with a tail
    tails = {g: len(t) % b for g, t in groups.items() if len(t) % b > 0} if stages >= 2 else {}
    keys = sorted(tails)
    nn = {}
    for g in keys:
        best, bd = None, None
        for h in keys:
            if h == g:
                continue
            dist = int(np.count_nonzero(masks[g] != masks[h]))
            if bd is None or dist < bd:
                best, bd = h, dist
        nn[g] = best
    pairs = []
    for g in keys:
        h = nn[g]
        if h is not None and g < h and nn.get(h) == g and tails[g] + tails[h] <= b:
            moved = groups[h][len(groups[h]) - tails[h]:]
            groups[h] = groups[h][:len(groups[h]) - tails[h]]
            groups[g] = groups[g] + moved
            new_masks[g] = masks[g] | masks[h]
            pairs.append((g, h, len(moved)))
    owner = np.full(labels_q.shape[0], -1, np.int32)
    for g, toks in groups.items():
        owner[np.asarray(toks, np.int64)] = g
    return owner, new_masks, groups, pairs


def dense_weights(q16: np.ndarray, K16h: np.ndarray, scale: float | None = None) -> np.ndarray:
    K16h = _c(K16h, np.uint16)
    L, d = K16h.shape
    w = np.empty(L, np.float64)
    sc = 1.0 / np.sqrt(d) if scale is None else scale
    lib().or_dense_weights(_p(_c(q16, np.uint16)), _p(K16h), ctypes.c_int(L), ctypes.c_int(d),
                           ctypes.c_double(sc), _p(w))
    return w


@dataclasses.dataclass
class LayerResult:
    labels_q: np.ndarray
    Cq: np.ndarray
    counts_q: np.ndarray
    kc: KClusters
    st: KStats
    S: list
    sel: list
    k: np.ndarray
    O: np.ndarray | None      # [BH, L, d] fp64 (None when attention is skipped)


def layer(Q16, K16, V16, p: Params, warm_from: LayerResult | None = None,
          attention: bool = True, rows=None) -> LayerResult:
    """One layer forward (Algorithm 3) for every head.  Q16/K16/V16: [BH, L, d]
    bf16 bits.  warm_from: the previous denoising step's result (warm start).
    rows: optional list of query rows to evaluate attention for (all if None)."""
    Q16 = _c(Q16, np.uint16)
    BH, L, d = Q16.shape
    if warm_from is None:
        lq, Cq, cq = cluster_q(Q16, p)
        kc = cluster_k_multistage(K16, p)
    else:
        lq, Cq, cq = cluster_q(Q16, p, init=warm_from.Cq, iters=p.iters_warm)
        kc = cluster_k_warm(K16, p, warm_from.kc)
    st = key_stats(K16, kc)
    S, sel, k = score_select(Cq, st, kc.n_k, p.topk, p.score_mode, kc.C)
    O = None
    if attention:
        r = np.arange(L) if rows is None else np.asarray(rows)
        O = np.empty((BH, r.size, d), np.float64)
        for h in range(BH):
            lab, sl = lq[h], sel[h]
            if p.tail_merge and not kc.F[h]:
                lab, sl = merged_selection(lq[h], sel[h], int(kc.n_k[h]), p.tail_merge)
            if p.compensate and not kc.F[h]:
                nk = int(kc.n_k[h])
                km, cnt = cluster_means(K16[h], kc.labels[h], nk)
                vm, _ = cluster_means(V16[h], kc.labels[h], nk)
                O[h] = attention_rows_comp(Q16[h], K16[h], V16[h], lab, kc.labels[h], sl, False, r, nk, cnt,
                                           km.astype(np.float64), vm.astype(np.float64))
            else:
                O[h] = attention_rows(Q16[h], K16[h], V16[h], lab, kc.labels[h], sl, bool(kc.F[h]), r)
    return LayerResult(lq, Cq, cq, kc, st, S, sel, k, O)


def merged_selection(labels_q, sel, nk: int, mode: int, b: int = 128):
    """The per-token attention sets after tail merging (mode 1: stage 1 only, 2:
    both stages) of one head: (owner per token, each owner's key clusters as
    rows padded with -1)."""
    Cq = sel.shape[0]
    masks = np.zeros((Cq, nk), bool)
    for q in range(Cq):
        masks[q, sel[q]] = True
    owner, new_masks, _, _ = tail_merge(labels_q, masks, b, stages=2 if mode >= 2 else 1)
    width = int(new_masks.sum(1).max())
    out = np.full((Cq, max(width, 1)), -1, np.int32)
    for q in range(Cq):
        c = np.nonzero(new_masks[q])[0]
        out[q, :c.size] = c
    return owner, out
