"""Python binding of libac over torch tensors (device memory and streams only).

Every call forwards torch data pointers and the current CUDA stream to the C
ABI in include/ac.h; all arithmetic of the layer runs in libac's kernels.
"""
from __future__ import annotations

import ctypes

import torch

from . import _lib
from ._lib import ACConfig, ACStageTimes, ACAttnCounters, check

_TORCH_DTYPES = {"<f4": torch.float32, "<i4": torch.int32, "|u1": torch.uint8, "<i2": torch.int16}


class _CudaArray:
    def __init__(self, ptr: int, shape, typestr: str):
        self.__cuda_array_interface__ = {"shape": tuple(shape), "typestr": typestr,
                                         "data": (int(ptr), False), "version": 3, "strides": None}


def _ptr(t):
    if t is None:
        return None
    if not t.is_contiguous():
        raise ValueError("tensors must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _bits(t):
    """bf16 tensor -> pointer to its uint16 bit patterns."""
    if t.dtype != torch.bfloat16:
        raise TypeError("Q, K, V, O must be torch.bfloat16")
    return _ptr(t)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def cluster_q_noalloc(Q, Cq: int, labels, centroids, iters: int = 10, seed: int = 1234, init=None, err=None):
    """ac_cluster_q_noalloc: angular k-means of Q [B, H, L, d] (bf16, CUDA) into
    caller-provided labels [B, H, L] int32 and centroids [B, H, Cq, d] fp32,
    with no device allocation inside the library (see include/ac.h).  err: an
    optional one-element int32 CUDA tensor that receives the kernels' error
    bits (1: a bounded wait expired, 4: non-finite input)."""
    lib = _lib.load()
    B, H, L, d = Q.shape
    check(lib.ac_cluster_q_noalloc(_bits(Q), B * H, L, d, Cq, iters, seed & (2**64 - 1), _ptr(init),
                                   _ptr(labels), _ptr(centroids), _ptr(err), _stream()))


def tau_exchange_allreduce(group=None, device=None):
    """An exchange function for SparseLayer.set_tau_exchange that sums the
    partial results over the ranks of a torch.distributed process group
    (all-reduce; NCCL over NVLink when device is a CUDA device, gloo on CPU)."""
    import torch.distributed as dist

    def fn(vals):
        t = torch.as_tensor(vals.astype("int64"), device=device or "cpu")
        dist.all_reduce(t, op=dist.ReduceOp.SUM, group=group)
        vals[:] = t.cpu().numpy().astype(vals.dtype)
    return fn


def calibrate_n_max(fallback_at, dense_frac: float = 0.15) -> int:
    """ac_calibrate_n_max: the N_max under which the ceil(dense_frac * n) units
    (of a stack of layers) with the largest AC_T_FALLBACK_AT fall back to dense
    attention (AdaCluster Sec. 4.1: the top 15% of layers run full attention)."""
    vals = [int(x) for x in fallback_at]
    arr = (ctypes.c_int32 * len(vals))(*vals)
    out = ctypes.c_int32(0)
    check(_lib.load().ac_calibrate_n_max(arr, len(vals), float(dense_frac), ctypes.byref(out)))
    return int(out.value)


def tau_mean_from_sums(factor: float, fixed_sum: int, n: int) -> float:
    """ac_tau_mean_from_sums: tau = factor x the mean of the pooled distances,
    from the sum of floor(d_i 2^24) and their number."""
    out = ctypes.c_float(0.0)
    check(_lib.load().ac_tau_mean_from_sums(float(factor), int(fixed_sum), int(n), ctypes.byref(out)))
    return float(out.value)


def tau_radix_pick(hist, shift: int, state):
    """ac_tau_radix_pick on a 256-bin summed histogram (sequence of ints) and the
    selection state [prefix, mask, rank] (updated and returned)."""
    h = (ctypes.c_uint64 * 256)(*[int(x) for x in hist])
    st = (ctypes.c_uint32 * 3)(*[int(x) for x in state])
    check(_lib.load().ac_tau_radix_pick(h, int(shift), st))
    return [int(st[0]), int(st[1]), int(st[2])]


class SparseLayer:
    """One cluster-routed sparse attention layer context for [B, H, L, d] inputs.

    Hyper-parameters follow ac_config in include/ac.h.  The context owns its
    workspace and the warm-start state carried across denoising steps."""

    def __init__(self, B: int, H: int, L: int, d: int, *, Cq: int, m0: int, n_max: int,
                 tau_mode: int, tau_value: float, topk: int, iters_q: int = 10,
                 iters_k: int = 10, iters_warm: int = 2, seed: int = 1234, scale: float = 0.0,
                 stage_rule: int = 0, score_mode: int = 0, tail_merge: int = 0, unit0: int = 0,
                 compensate: int = 0):
        self.lib = _lib.load()
        self.B, self.H, self.L, self.d = B, H, L, d
        self.cfg = ACConfig(Cq, m0, n_max, tau_mode, float(tau_value), topk, iters_q, iters_k,
                            iters_warm, stage_rule, seed & (2**64 - 1), float(scale), score_mode,
                            tail_merge, unit0, compensate)
        self.Cq, self.Ccap = Cq, n_max + m0
        h = ctypes.c_void_p()
        check(self.lib.ac_create(ctypes.byref(self.cfg), B, H, L, d, ctypes.byref(h)))
        self.ctx = h

    @classmethod
    def from_config(cls, cfg, seed: int = 1234, B=None, H=None, L=None, **kw):
        """Build from a synth.LayerConfig (shape overrides allowed; keyword
        arguments such as score_mode or tail_merge are passed on)."""
        return cls(B or cfg.B, H or cfg.H, L or cfg.L, cfg.d, Cq=cfg.Cq, m0=cfg.m0, n_max=cfg.n_max,
                   tau_mode=cfg.tau_mode, tau_value=cfg.tau_value, topk=cfg.topk,
                   iters_q=cfg.iters_q, iters_k=cfg.iters_k, iters_warm=cfg.iters_warm, seed=seed,
                   stage_rule=cfg.stage_rule, **kw)

    def set_tau_exchange(self, fn):
        """Pool tau with other contexts that hold the other heads of the layer:
        fn(vals) receives a numpy uint64 array of partial sums and must replace
        it, in place, by the sums over all contexts (see ac_set_tau_exchange);
        None: tau from this context's heads."""
        import numpy as np
        if fn is None:
            self._xchg = None
            check(self.lib.ac_set_tau_exchange(self.ctx, _lib.SUM_U64_FN(), None), self.ctx)
            return

        def cb(_user, data, count):
            try:
                vals = np.ctypeslib.as_array(data, shape=(count,))
                fn(vals)
                return 0
            except Exception:  # reported to the library as a failed exchange
                return 1
        self._xchg = _lib.SUM_U64_FN(cb)  # kept alive with the context
        check(self.lib.ac_set_tau_exchange(self.ctx, self._xchg, None), self.ctx)

    # ------------------------------------------------------------------ calls
    def cluster_q(self, Q, init=None, iters: int = -1, labels=None, centroids=None):
        check(self.lib.ac_cluster_q(self.ctx, _bits(Q), _ptr(init), iters, _ptr(labels),
                                    _ptr(centroids), _stream()), self.ctx)

    def cluster_k(self, K, warm_centroids=None, warm_n_k=None, warm_dense=None, labels=None,
                  centroids=None, n_k=None, dense=None, comp=None):
        check(self.lib.ac_cluster_k_multistage(
            self.ctx, _bits(K), _ptr(warm_centroids), _ptr(warm_n_k), _ptr(warm_dense),
            _ptr(labels), _ptr(centroids), _ptr(n_k), _ptr(dense), _ptr(comp), _stream()), self.ctx)

    def score_select(self, topk: int = 0, sel=None, k=None):
        check(self.lib.ac_score_select(self.ctx, topk, _ptr(sel), _ptr(k), _stream()), self.ctx)

    def sparse_attn(self, Q, K, V, O=None):
        if O is None:
            O = torch.empty_like(Q)
        check(self.lib.ac_sparse_attn(self.ctx, _bits(Q), _bits(K), _bits(V), _bits(O), _stream()),
              self.ctx)
        return O

    def forward(self, Q, K, V, O=None, warm: bool = False, times: bool = False):
        if O is None:
            O = torch.empty_like(Q)
        t = ACStageTimes() if times else None
        check(self.lib.ac_layer_forward(self.ctx, _bits(Q), _bits(K), _bits(V), _bits(O),
                                        1 if warm else 0, ctypes.byref(t) if t is not None else None,
                                        _stream()), self.ctx)
        return (O, t.as_dict()) if times else O

    def forward_host(self, hQ, hK, hV, hO, warm: bool = False):
        """Host (ideally pinned) bf16 tensors in and out; copies inside the call."""
        check(self.lib.ac_layer_forward_host(self.ctx, _bits(hQ), _bits(hK), _bits(hV), _bits(hO),
                                             1 if warm else 0, _stream()), self.ctx)
        return hO

    def forward_host_async(self, hQ, hK, hV, hO, warm: bool = False):
        """As forward_host, without waiting: hO is written once the current
        stream has passed join() (or after synchronize()); keep the inputs
        unchanged until then.  Consecutive calls overlap their copies with the
        neighbouring calls' layers."""
        check(self.lib.ac_layer_forward_host_async(self.ctx, _bits(hQ), _bits(hK), _bits(hV), _bits(hO),
                                                   1 if warm else 0, _stream()), self.ctx)
        return hO

    def join(self):
        """Make the current stream wait for the output copies of earlier async calls."""
        check(self.lib.ac_join(self.ctx, _stream()), self.ctx)

    def synchronize(self):
        check(self.lib.ac_synchronize(self.ctx, _stream()), self.ctx)

    def check_wait_timeout(self, limit_us: int):
        """Enqueue the bounded-wait health check (ac_check_wait_timeout); the
        next synchronize() raises with AC_ERR_TIMEOUT."""
        check(self.lib.ac_check_wait_timeout(self.ctx, int(limit_us), _stream()), self.ctx)

    def tensor(self, which: int) -> torch.Tensor:
        """Device view of an intermediate tensor (ac_get_tensor); valid until the next call."""
        p = ctypes.c_void_p()
        shape = (ctypes.c_int64 * 4)()
        check(self.lib.ac_get_tensor(self.ctx, which, ctypes.byref(p), shape), self.ctx)
        typ = _lib.TENSOR_TYPES[which]
        dims = [int(x) for x in shape[:_lib.TENSOR_RANKS[which]]]
        t = torch.as_tensor(_CudaArray(p.value, dims, typ), device="cuda")
        if which in (_lib.AC_T_KMAX, _lib.AC_T_KMIN):
            t = t.view(torch.bfloat16)
        return t

    def launch_count(self) -> int:
        """Kernels libac has launched in this process so far."""
        n = ctypes.c_int64(0)
        check(self.lib.ac_get_launch_count(ctypes.byref(n)), self.ctx)
        return int(n.value)

    def counters(self) -> dict:
        c = ACAttnCounters()
        check(self.lib.ac_get_attn_counters(self.ctx, ctypes.byref(c)), self.ctx)
        return {f: int(getattr(c, f)) for f, _ in c._fields_}

    def assign_counters(self, reset: bool = False) -> dict:
        """Tensor-core / exact assignment passes and rows rescored exactly."""
        c = _lib.ACAssignCounters()
        check(self.lib.ac_get_assign_counters(self.ctx, ctypes.byref(c), 1 if reset else 0), self.ctx)
        return {f: int(getattr(c, f)) for f, _ in c._fields_}

    def export_state(self) -> bytes:
        n = ctypes.c_int64(0)
        check(self.lib.ac_state_export(self.ctx, None, ctypes.byref(n)), self.ctx)
        buf = ctypes.create_string_buffer(n.value)
        check(self.lib.ac_state_export(self.ctx, buf, ctypes.byref(n)), self.ctx)
        return buf.raw

    def import_state(self, data: bytes):
        buf = ctypes.create_string_buffer(data, len(data))
        check(self.lib.ac_state_import(self.ctx, buf, len(data)), self.ctx)

    def close(self):
        if getattr(self, "ctx", None):
            self.lib.ac_destroy(self.ctx)
            self.ctx = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass
