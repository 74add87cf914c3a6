"""ctypes declarations of the libac C ABI (include/ac.h).

Argument marshalling only: every step of the layer runs in libac's kernels.
Loading fails loudly when libac.so has not been built; there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libac.so")

AC_OK, AC_ERR_INVALID_ARG, AC_ERR_UNSUPPORTED, AC_ERR_WORKSPACE, AC_ERR_CUDA, \
    AC_ERR_NONFINITE, AC_ERR_TIMEOUT, AC_ERR_STATE = range(8)
STATUS_NAMES = ["AC_OK", "AC_ERR_INVALID_ARG", "AC_ERR_UNSUPPORTED", "AC_ERR_WORKSPACE", "AC_ERR_CUDA",
                "AC_ERR_NONFINITE", "AC_ERR_TIMEOUT", "AC_ERR_STATE"]

AC_TAU_ABSOLUTE, AC_TAU_MEAN_FACTOR, AC_TAU_PERCENTILE = 0, 1, 2

# ac_tensor_id
(AC_T_INV_NORM_Q, AC_T_LABELS_Q, AC_T_CENT_Q, AC_T_COUNTS_Q, AC_T_PERM_Q, AC_T_OFFS_Q, AC_T_LABELS_K,
 AC_T_DMIN_K, AC_T_CENT_K, AC_T_N_K, AC_T_DENSE, AC_T_COUNTS_K, AC_T_KMAX, AC_T_KMIN, AC_T_SSE, AC_T_COMP,
 AC_T_PERM_K, AC_T_OFFS_K, AC_T_SCORE, AC_T_SEL, AC_T_KSEL, AC_T_TAU, AC_T_STAGES, AC_T_REMOVED_STAGE,
 AC_T_MSE, AC_T_FALLBACK_AT) = range(26)

# element type of each tensor id, as a __cuda_array_interface__ typestr
TENSOR_TYPES = {
    AC_T_INV_NORM_Q: "<f4", AC_T_LABELS_Q: "<i4", AC_T_CENT_Q: "<f4", AC_T_COUNTS_Q: "<i4",
    AC_T_PERM_Q: "<i4", AC_T_OFFS_Q: "<i4", AC_T_LABELS_K: "<i4", AC_T_DMIN_K: "<f4",
    AC_T_CENT_K: "<f4", AC_T_N_K: "<i4", AC_T_DENSE: "|u1", AC_T_COUNTS_K: "<i4", AC_T_KMAX: "<i2",
    AC_T_KMIN: "<i2", AC_T_SSE: "<f4", AC_T_COMP: "<f4", AC_T_PERM_K: "<i4", AC_T_OFFS_K: "<i4",
    AC_T_SCORE: "<f4", AC_T_SEL: "<i4", AC_T_KSEL: "<i4", AC_T_TAU: "<f4", AC_T_STAGES: "<i4",
    AC_T_REMOVED_STAGE: "<i4", AC_T_MSE: "<f4", AC_T_FALLBACK_AT: "<i4",
}


# rank of each tensor id (ac_get_tensor reports unused trailing extents as 1)
TENSOR_RANKS = {
    AC_T_INV_NORM_Q: 2, AC_T_LABELS_Q: 2, AC_T_CENT_Q: 3, AC_T_COUNTS_Q: 2, AC_T_PERM_Q: 2,
    AC_T_OFFS_Q: 2, AC_T_LABELS_K: 2, AC_T_DMIN_K: 2, AC_T_CENT_K: 3, AC_T_N_K: 1, AC_T_DENSE: 1,
    AC_T_COUNTS_K: 2, AC_T_KMAX: 3, AC_T_KMIN: 3, AC_T_SSE: 2, AC_T_COMP: 1, AC_T_PERM_K: 2,
    AC_T_OFFS_K: 2, AC_T_SCORE: 3, AC_T_SEL: 3, AC_T_KSEL: 1, AC_T_TAU: 1, AC_T_STAGES: 1,
    AC_T_REMOVED_STAGE: 2, AC_T_MSE: 1, AC_T_FALLBACK_AT: 1,
}


class ACConfig(ctypes.Structure):
    _fields_ = [("Cq", ctypes.c_int32), ("m0", ctypes.c_int32), ("n_max", ctypes.c_int32),
                ("tau_mode", ctypes.c_int32), ("tau_value", ctypes.c_float), ("topk", ctypes.c_int32),
                ("iters_q", ctypes.c_int32), ("iters_k", ctypes.c_int32), ("iters_warm", ctypes.c_int32),
                ("stage_rule", ctypes.c_int32), ("seed", ctypes.c_uint64), ("scale", ctypes.c_float),
                ("score_mode", ctypes.c_int32), ("tail_merge", ctypes.c_int32), ("unit0", ctypes.c_int32),
                ("compensate", ctypes.c_int32)]


class ACStageTimes(ctypes.Structure):
    _fields_ = [("q_cluster_ms", ctypes.c_float), ("k_cluster_ms", ctypes.c_float),
                ("stats_sort_ms", ctypes.c_float), ("score_select_ms", ctypes.c_float),
                ("attention_ms", ctypes.c_float), ("attn_kernel_ms", ctypes.c_float),
                ("total_ms", ctypes.c_float)]

    def as_dict(self):
        return {f: float(getattr(self, f)) for f, _ in self._fields_}


class ACAttnCounters(ctypes.Structure):
    _fields_ = [("kept_pairs", ctypes.c_int64), ("computed_pairs", ctypes.c_int64),
                ("tiles", ctypes.c_int64), ("dense_heads", ctypes.c_int64),
                ("wait_failure", ctypes.c_int64)]


class ACAssignCounters(ctypes.Structure):
    _fields_ = [("tensor_passes", ctypes.c_int64), ("exact_passes", ctypes.c_int64),
                ("rows", ctypes.c_int64), ("uncertain_rows", ctypes.c_int64),
                ("full_rescore_rows", ctypes.c_int64)]


# every function that include/ac.h declares, with its ctypes signature
_P = ctypes.c_void_p
_I = ctypes.c_int32
# int32_t (*ac_sum_u64_fn)(void *user, uint64_t *data, int32_t count)
SUM_U64_FN = ctypes.CFUNCTYPE(ctypes.c_int32, ctypes.c_void_p, ctypes.POINTER(ctypes.c_uint64), ctypes.c_int32)
SIGNATURES = {
    "ac_create": (_I, [ctypes.POINTER(ACConfig), _I, _I, _I, _I, ctypes.POINTER(_P)]),
    "ac_destroy": (_I, [_P]),
    "ac_last_error_string": (ctypes.c_char_p, [_P]),
    "ac_cluster_q": (_I, [_P, _P, _P, _I, _P, _P, _P]),
    "ac_cluster_k_multistage": (_I, [_P, _P, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "ac_score_select": (_I, [_P, _I, _P, _P, _P]),
    "ac_sparse_attn": (_I, [_P, _P, _P, _P, _P, _P]),
    "ac_layer_forward": (_I, [_P, _P, _P, _P, _P, _I, ctypes.POINTER(ACStageTimes), _P]),
    "ac_layer_forward_host": (_I, [_P, _P, _P, _P, _P, _I, _P]),
    "ac_layer_forward_host_async": (_I, [_P, _P, _P, _P, _P, _I, _P]),
    "ac_join": (_I, [_P, _P]),
    "ac_synchronize": (_I, [_P, _P]),
    "ac_check_wait_timeout": (_I, [_P, ctypes.c_int32, _P]),
    "ac_get_tensor": (_I, [_P, _I, ctypes.POINTER(_P), ctypes.POINTER(ctypes.c_int64)]),
    "ac_get_attn_counters": (_I, [_P, ctypes.POINTER(ACAttnCounters)]),
    "ac_get_launch_count": (_I, [ctypes.POINTER(ctypes.c_int64)]),
    "ac_get_assign_counters": (_I, [_P, ctypes.POINTER(ACAssignCounters), _I]),
    "ac_cluster_q_noalloc": (_I, [_P, _I, _I, _I, _I, _I, ctypes.c_uint64, _P, _P, _P, _P, _P]),
    "ac_state_export": (_I, [_P, _P, ctypes.POINTER(ctypes.c_int64)]),
    "ac_set_tau_exchange": (_I, [_P, SUM_U64_FN, _P]),
    "ac_calibrate_n_max": (_I, [ctypes.POINTER(_I), ctypes.c_int64, ctypes.c_float, ctypes.POINTER(_I)]),
    "ac_tau_mean_from_sums": (_I, [ctypes.c_float, ctypes.c_uint64, ctypes.c_uint64, ctypes.POINTER(ctypes.c_float)]),
    "ac_tau_radix_pick": (_I, [ctypes.POINTER(ctypes.c_uint64), _I, ctypes.POINTER(ctypes.c_uint32)]),
    "ac_state_import": (_I, [_P, _P, ctypes.c_int64]),
}

_lib = None


def load() -> ctypes.CDLL:
    """Load libac.so (raises if it is missing: there is no CPU path)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"libac.so is not built ({LIB_PATH}); run "
                               "`python -m cluster_routed_sparse_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib


class ACError(RuntimeError):
    def __init__(self, status: int, msg: str):
        self.status = status
        name = STATUS_NAMES[status] if 0 <= status < len(STATUS_NAMES) else str(status)
        super().__init__(f"{name}: {msg}")


def check(status: int, ctx=None) -> None:
    if status != AC_OK:
        msg = load().ac_last_error_string(ctx)
        raise ACError(status, msg.decode() if msg else "")
