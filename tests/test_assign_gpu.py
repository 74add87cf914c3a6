"""GPU checks of the tensor-core k-means assignment (split centres, error
bound, exact rescoring of the rows the bound cannot settle).

The labels must equal those of the exact fp32 definition: against the oracle
on inputs built to produce exact ties and large magnitudes, and against the
library's own exact CUDA-core kernel (AC_EXACT_ASSIGN=1) at a size with
several centre chunks per row tile.
"""
import os

import numpy as np
import pytest
import torch

from _gpu_common import compare_layer, dev, gpu_state, make_layer_ctx, run_gpu_layer
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def _flat(x):
    B, H, L, d = x.shape
    return x.reshape(B * H, L, d)


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return synth.f32_to_bf16_bits(np.ascontiguousarray(x, np.float32))


def test_duplicate_tokens_tie_to_lowest_index():
    """96 distinct rows, each repeated 16 times: seeds coincide, so centres
    coincide and distances tie exactly; the lowest centre index must win."""
    rng = np.random.default_rng(11)
    B, H, L, d = 1, 2, 1536, 128
    base_q = rng.standard_normal((H, 96, d)).astype(np.float32)
    base_k = rng.standard_normal((H, 96, d)).astype(np.float32)
    idx = np.repeat(np.arange(96), 16)
    rng.shuffle(idx)
    Q = _bf16_bits(base_q[:, idx]).reshape(B, H, L, d)
    K = _bf16_bits(base_k[:, idx]).reshape(B, H, L, d)
    V = _bf16_bits(rng.standard_normal((B, H, L, d))).reshape(B, H, L, d)
    cfg = synth.LayerConfig("dup", B, H, L, d, Cq=40, m0=48, n_max=200, tau_mode=1, tau_value=1.0, topk=-200,
                            iters_q=4, iters_k=4)
    p = orc.Params.from_layer_config(cfg, seed=5)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    c = lay.assign_counters()
    assert c["tensor_passes"] > 0
    assert c["uncertain_rows"] > 0, c  # exact ties can only be settled by rescoring
    lay.close()


def test_large_magnitude_keys():
    """Keys scaled by 2^6 (exact in bf16): |k|^2 ~ 5e5, distances far from 1."""
    cfg = synth.LayerConfig("big", 1, 2, 2500, 128, Cq=20, m0=40, n_max=160, tau_mode=1, tau_value=1.0,
                            topk=-150, key_components=40, iters_q=3, iters_k=3)
    Q, K, V = synth.make_layer(cfg)
    Kf = synth.bf16_bits_to_f32(K) * np.float32(64.0)
    K = _bf16_bits(Kf).reshape(K.shape)
    p = orc.Params.from_layer_config(cfg, seed=8)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def _run_two_steps(cfg, p, exact: bool):
    old = os.environ.get("AC_EXACT_ASSIGN")
    os.environ["AC_EXACT_ASSIGN"] = "1" if exact else "0"
    try:
        lay = make_layer_ctx(p, cfg.B, cfg.H, cfg.L, cfg.d)
    finally:
        if old is None:
            del os.environ["AC_EXACT_ASSIGN"]
        else:
            os.environ["AC_EXACT_ASSIGN"] = old
    states = []
    for step in range(2):
        Q, K, V = synth.make_layer(cfg, step=step)
        lay, O, gs = run_gpu_layer(Q, K, V, p, lay=lay, warm=step > 0)
        states.append((gs, O))
    return lay, states


def test_tensor_core_assignment_equals_exact_kernel():
    """Several 256-centre chunks per row tile (n_max + m0 = 1256), step 0 and
    one warm step: every label, centre and output identical to the exact
    kernel's."""
    cfg = synth.LayerConfig("chunks", 1, 4, 16384, 128, Cq=65, m0=256, n_max=1000, tau_mode=1, tau_value=1.5,
                            topk=-100, key_components=400, iters_q=4, iters_k=3)
    p = orc.Params.from_layer_config(cfg, seed=21)
    p.iters_warm = 2
    lay_f, st_f = _run_two_steps(cfg, p, exact=False)
    lay_e, st_e = _run_two_steps(cfg, p, exact=True)
    cf, ce = lay_f.assign_counters(), lay_e.assign_counters()
    assert cf["tensor_passes"] > 0 and ce["tensor_passes"] == 0, (cf, ce)
    assert cf["uncertain_rows"] < 0.25 * cf["rows"], cf
    for step, ((gf, Of), (ge, Oe)) in enumerate(zip(st_f, st_e)):
        for k in ("labels_q", "labels_k", "n_k", "dense", "perm_q", "perm_k", "ksel", "stages", "removed_stage"):
            np.testing.assert_array_equal(gf[k], ge[k], err_msg=f"step {step}: {k}")
        for k in ("cent_q", "cent_k", "dmin_k", "sse", "tau"):
            np.testing.assert_array_equal(gf[k], ge[k], err_msg=f"step {step}: {k}")
        np.testing.assert_array_equal(Of, Oe, err_msg=f"step {step}: output")
    lay_f.close()
    lay_e.close()
