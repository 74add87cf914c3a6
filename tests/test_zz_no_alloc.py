"""The allocation-free query clustering entry point (ac_cluster_q_noalloc),
called through the C ABI, gives the same labels and centres as ac_cluster_q,
on two calls in a row (its scratch array keeps the previous call's contents).

It serves callers that cannot allocate device memory while they run (for
example an inference engine's plugin callback), so its scratch is a fixed
__device__ array inside the library instead of a context workspace."""
import ctypes

import numpy as np
import pytest
import torch

from _gpu_common import CENT_RTOL, dev, make_layer_ctx
from oracle import oracle as orc
from cluster_routed_sparse_b200 import _lib, synth

pytestmark = pytest.mark.gpu


def _noalloc(lib, Q, Cq, iters, seed, labels, cent, init=None, err=None):
    B, H, L, d = Q.shape
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    return lib.ac_cluster_q_noalloc(ctypes.c_void_p(Q.data_ptr()), B * H, L, d, Cq, iters, seed,
                                    ctypes.c_void_p(init.data_ptr()) if init is not None else None,
                                    ctypes.c_void_p(labels.data_ptr()), ctypes.c_void_p(cent.data_ptr()),
                                    ctypes.c_void_p(err.data_ptr()) if err is not None else None, stream)


@pytest.mark.parametrize("cfg", [synth.CONFIGS[1],
                                 synth.LayerConfig("noalloc-d128", 1, 3, 3000, 128, Cq=11, m0=8, n_max=16,
                                                   tau_mode=1, tau_value=1.0, topk=2, iters_q=5)])
def test_noalloc_matches_cluster_q_on_two_calls(cfg):
    lib = _lib.load()
    Q16, _, _ = synth.make_layer(cfg)
    Q = dev(Q16)
    p = orc.Params.from_layer_config(cfg, seed=4321)
    lay = make_layer_ctx(p, cfg.B, cfg.H, cfg.L, cfg.d)
    BH = cfg.B * cfg.H
    ref_lab = torch.empty((BH, cfg.L), dtype=torch.int32, device="cuda")
    ref_cent = torch.empty((BH, cfg.Cq, cfg.d), dtype=torch.float32, device="cuda")
    lay.cluster_q(Q, labels=ref_lab, centroids=ref_cent)
    torch.cuda.synchronize()
    for call in range(2):
        lab = torch.full((BH, cfg.L), -7, dtype=torch.int32, device="cuda")
        cent = torch.full((BH, cfg.Cq, cfg.d), float("nan"), dtype=torch.float32, device="cuda")
        err = torch.full((1,), 99, dtype=torch.int32, device="cuda")  # the call clears it
        st = _noalloc(lib, Q, cfg.Cq, cfg.iters_q, p.seed, lab, cent, err=err)
        assert st == _lib.AC_OK, lib.ac_last_error_string(None)
        torch.cuda.synchronize()
        assert int(err.item()) == 0, f"kernel error bits {int(err.item())} on call {call}"
        assert torch.equal(lab, ref_lab), f"labels differ on call {call}"
        err = (cent.double() - ref_cent.double()).abs()
        tol = CENT_RTOL * ref_cent.double().abs().clamp_min(1e-3)
        assert bool((err <= tol).all()), f"centres differ on call {call}"
    lay.close()


def test_noalloc_warm_start_and_limits():
    lib = _lib.load()
    cfg = synth.CONFIGS[1]
    Q16, _, _ = synth.make_layer(cfg)
    Q = dev(Q16)
    p = orc.Params.from_layer_config(cfg, seed=11)
    lay = make_layer_ctx(p, cfg.B, cfg.H, cfg.L, cfg.d)
    BH = cfg.B * cfg.H
    init = torch.empty((BH, cfg.Cq, cfg.d), dtype=torch.float32, device="cuda")
    lab0 = torch.empty((BH, cfg.L), dtype=torch.int32, device="cuda")
    lay.cluster_q(Q, labels=lab0, centroids=init)           # step 0 centres
    ref_lab = torch.empty_like(lab0)
    ref_cent = torch.empty_like(init)
    lay.cluster_q(Q, init=init, iters=2, labels=ref_lab, centroids=ref_cent)  # warm step
    lab = torch.empty_like(lab0)
    cent = torch.empty_like(init)
    assert _noalloc(lib, Q, cfg.Cq, 2, 0, lab, cent, init=init) == _lib.AC_OK
    torch.cuda.synchronize()
    assert torch.equal(lab, ref_lab) and torch.equal(cent, ref_cent)
    # beyond the stated maximum: rejected before any work, with a message
    big = torch.empty((1, 1, 1, 64), dtype=torch.bfloat16, device="cuda")
    st = lib.ac_cluster_q_noalloc(ctypes.c_void_p(big.data_ptr()), 1 << 11, 1 << 10, 64, 4, 1, 0, None,
                                  ctypes.c_void_p(lab.data_ptr()), ctypes.c_void_p(cent.data_ptr()), None, None)
    assert st == _lib.AC_ERR_INVALID_ARG
    assert b"1048576" in lib.ac_last_error_string(None)
    # more centres than the sort's shared-memory histograms hold: rejected up front too
    st = lib.ac_cluster_q_noalloc(ctypes.c_void_p(big.data_ptr()), 1, 8192, 64, 4097, 1, 0, None,
                                  ctypes.c_void_p(lab.data_ptr()), ctypes.c_void_p(cent.data_ptr()), None, None)
    assert st == _lib.AC_ERR_INVALID_ARG
    assert b"4096" in lib.ac_last_error_string(None)
    lay.close()
