"""GPU parity: the CUDA layer (through the C ABI) against the CPU oracle.

Labels, permutations, stage bookkeeping and selections are compared
bit-exactly, centres within fp32 relative 1e-4, and the attention output
within max abs 2e-2 / relative L2 5e-3 of the fp64 oracle.
"""
import numpy as np
import pytest
import torch

from _gpu_common import (assert_attention, compare_layer, dev, gpu_state, heavy_tail_layer, host_f32,
                         make_layer_ctx, run_gpu_layer)
from oracle import oracle as orc
from cluster_routed_sparse_b200 import synth

pytestmark = pytest.mark.gpu


def _params(cfg, seed=1234, **kw):
    p = orc.Params.from_layer_config(cfg, seed=seed)
    for k, v in kw.items():
        setattr(p, k, v)
    return p


def _flat(x):
    B, H, L, d = x.shape
    return x.reshape(B * H, L, d)


def test_tiny_layer_step0_end_to_end():
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_mean_score_ablation_end_to_end():
    """score_mode 1 (the "w/o Quest" ablation, Sec. 4.4 Table 4): key clusters
    scored by q . centre; scores, selections and outputs against the oracle."""
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg, score_mode=1)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    # the ablation changes what is kept
    r0 = orc.layer(_flat(Q), _flat(K), _flat(V), _params(cfg), attention=False)
    assert any(not np.array_equal(a, b) for a, b in zip(r.sel, r0.sel))
    lay.close()


@pytest.mark.parametrize("mode", [1, 2])
def test_tail_merge_end_to_end(mode):
    """ac_config.tail_merge (iCATS tail merging of the query tiles): query
    clusters with the same selection share tiles (mode 1; four of the sixteen
    clusters fold in here), and mutually nearest clusters with small tails pool
    them (mode 2; three pairs here); outputs against the oracle's per-token key
    sets after the same merge."""
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg, tail_merge=mode)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_tail_merge_dense_units():
    """Every unit dense: every query cluster walks every key, so stage 1 folds
    all of them into one group; the output stays dense attention."""
    cfg = synth.LayerConfig("dense", 1, 2, 1200, 64, Cq=5, m0=8, n_max=20, tau_mode=0, tau_value=0.0,
                            topk=2, key_components=20, iters_q=3, iters_k=2)
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg, tail_merge=2)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    assert r.kc.F.all()
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_tiny_layer_warm_chain():
    """Step 0 then two warm-started steps on perturbed tokens (Sec. 3.2.2)."""
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    lay = None
    prev = None
    for step in range(3):
        Q, K, V = synth.make_layer(cfg, step=step)
        r = orc.layer(_flat(Q), _flat(K), _flat(V), p, warm_from=prev)
        lay, O, gs = run_gpu_layer(Q, K, V, p, lay=lay, warm=step > 0)
        compare_layer(gs, r, p, O, check_step0=step == 0)
        prev = r
    lay.close()


@pytest.mark.parametrize("shape,kw", [
    ((1, 2, 1000, 64), dict(Cq=7, m0=10, n_max=40, tau_mode=1, tau_value=1.0, topk=-300)),
    ((1, 2, 2048, 128), dict(Cq=16, m0=16, n_max=64, tau_mode=2, tau_value=900.0, topk=4)),
    ((2, 2, 1500, 64), dict(Cq=9, m0=12, n_max=48, tau_mode=1, tau_value=1.5, topk=-100)),
    ((1, 1, 333, 128), dict(Cq=3, m0=5, n_max=20, tau_mode=1, tau_value=1.2, topk=2)),
])
def test_ragged_shapes(shape, kw):
    B, H, Lq, d = shape
    cfg = synth.LayerConfig("ragged", B, H, Lq, d, key_components=30, iters_q=4, iters_k=4, **kw)
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg, seed=99)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_heavy_tailed_clusters():
    """Dirichlet(0.3) component weights: many clusters under 8 keys, so most
    key boxes are partly masked."""
    cfg = heavy_tail_layer()
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg, seed=7)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    assert (r.st.counts[:, :int(r.kc.n_k.min())] < 8).sum() > 0
    lay.close()


def test_dense_fallback_heads():
    """tau = 0 absorbs nothing: every head reaches N_max and attends densely
    (Algorithm 1 lines 7-9, Algorithm 3 line 6)."""
    cfg = synth.LayerConfig("dense", 1, 2, 1200, 64, Cq=5, m0=8, n_max=20, tau_mode=0, tau_value=0.0,
                            topk=2, key_components=20, iters_q=3, iters_k=2)
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    assert r.kc.F.all()
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_all_clusters_selected_is_dense_attention():
    cfg = synth.LayerConfig("allsel", 1, 2, 1536, 128, Cq=6, m0=12, n_max=40, tau_mode=1,
                            tau_value=1.0, topk=10000, key_components=25, iters_q=3, iters_k=3)
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    for h in range(2):
        ref = orc.attention_rows(Q[0, h], K[0, h], V[0, h], gs["labels_q"][h], gs["labels_k"][h],
                                 None, True, np.arange(cfg.L))
        assert_attention(O[h], ref, f"head {h}")
    lay.close()


@pytest.mark.parametrize("Lq", [1, 5, 9])
def test_tiny_sequences(Lq):
    cfg = synth.LayerConfig("tiny", 1, 1, Lq, 64, Cq=min(2, Lq), m0=min(3, Lq), n_max=4, tau_mode=1,
                            tau_value=1.0, topk=1, key_components=2, iters_q=2, iters_k=2)
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg)
    r = orc.layer(_flat(Q), _flat(K), _flat(V), p)
    lay, O, gs = run_gpu_layer(Q, K, V, p)
    compare_layer(gs, r, p, O)
    lay.close()


def test_host_entry_point_matches_device_forward():
    cfg = synth.CONFIGS[1]
    Q, K, V = synth.make_layer(cfg)
    p = _params(cfg)
    lay, O, _ = run_gpu_layer(Q, K, V, p)
    lay2 = make_layer_ctx(p, *Q.shape)
    hQ, hK, hV = (torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in (Q, K, V))
    hO = torch.empty_like(hQ).pin_memory()
    lay2.forward_host(hQ, hK, hV, hO)
    assert np.array_equal(hO.view(torch.int16).numpy().reshape(O.shape),
                          torch.from_numpy(O).to(torch.bfloat16).view(torch.int16).numpy())
    lay.close()
    lay2.close()


def test_async_host_entry_point_pipelines_three_steps():
    """ac_layer_forward_host_async over step 0 and two warm steps (calls queued
    back to back, copies overlapping the neighbouring layers) gives the same
    outputs as the device-buffer forward of the same steps."""
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    steps = [synth.make_layer(cfg, step=s) for s in range(3)]
    ref = make_layer_ctx(p, *steps[0][0].shape)
    want = []
    for s, (Q, K, V) in enumerate(steps):
        q, k, v = dev(Q), dev(K), dev(V)
        o = torch.empty_like(q)
        ref.forward(q, k, v, o, warm=s > 0)
        ref.synchronize()
        want.append(o.view(torch.int16).cpu().numpy())
    lay = make_layer_ctx(p, *steps[0][0].shape)
    host = [[torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in st] for st in steps]
    outs = [torch.empty_like(host[0][0]).pin_memory() for _ in steps]
    for s in range(3):
        lay.forward_host_async(*host[s], outs[s], warm=s > 0)
    lay.synchronize()
    for s in range(3):
        assert np.array_equal(outs[s].view(torch.int16).numpy(), want[s].reshape(outs[s].shape)), s
    ref.close()
    lay.close()


def test_state_resume_is_bit_exact():
    """Checkpoint/resume across denoising steps: exporting the warm-start state
    after step 0 and importing it into a fresh context gives the same warm step."""
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    Q0, K0, V0 = synth.make_layer(cfg, step=0)
    Q1, K1, V1 = synth.make_layer(cfg, step=1)
    a, _, _ = run_gpu_layer(Q0, K0, V0, p)
    blob = a.export_state()
    _, Oa, ga = run_gpu_layer(Q1, K1, V1, p, lay=a, warm=True)
    b = make_layer_ctx(p, *Q0.shape)
    b.import_state(blob)
    _, Ob, gb = run_gpu_layer(Q1, K1, V1, p, lay=b, warm=True)
    assert np.array_equal(Oa, Ob)
    for key in ("labels_q", "labels_k", "cent_q", "cent_k", "ksel"):
        assert np.array_equal(ga[key], gb[key]), key
    for h in range(ga["ksel"].shape[0]):
        k = int(ga["ksel"][h])
        assert np.array_equal(ga["sel"][h, :, :k], gb["sel"][h, :, :k])
    a.close()
    b.close()


def test_warm_step_before_step0_is_a_state_error():
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    lay = make_layer_ctx(p, 1, 2, cfg.L, cfg.d)
    Q, K, V = (dev(x) for x in synth.make_layer(cfg))
    from cluster_routed_sparse_b200._lib import ACError, AC_ERR_STATE
    with pytest.raises(ACError) as e:
        lay.forward(Q, K, V, warm=True)
    assert e.value.status == AC_ERR_STATE
    lay.close()


def test_nonfinite_input_is_reported():
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    Q, K, V = synth.make_layer(cfg)
    Q = Q.copy()
    Q[0, 0, 17, 3] = 0x7FC0  # bf16 NaN
    lay = make_layer_ctx(p, *Q.shape)
    from cluster_routed_sparse_b200._lib import ACError, AC_ERR_NONFINITE
    with pytest.raises(ACError) as e:
        lay.cluster_q(dev(Q))
    assert e.value.status == AC_ERR_NONFINITE
    lay.close()


def test_bounded_wait_timeout_is_reported_and_context_stays_usable():
    """A bounded in-kernel wait on a phase nothing completes ends after its
    limit with AC_ERR_TIMEOUT on the host; the context then runs the layer to
    the same output as before the timeout."""
    import time
    from cluster_routed_sparse_b200._lib import ACError, AC_ERR_TIMEOUT, AC_ERR_INVALID_ARG
    cfg = synth.CONFIGS[1]
    p = _params(cfg)
    Q, K, V = (dev(x) for x in synth.make_layer(cfg))
    lay = make_layer_ctx(p, *Q.shape)
    O0 = lay.forward(Q, K, V).clone()
    lay.synchronize()
    for bad in (0, -5, 2000001):
        with pytest.raises(ACError) as e:
            lay.check_wait_timeout(bad)
        assert e.value.status == AC_ERR_INVALID_ARG
    t0 = time.perf_counter()
    lay.check_wait_timeout(20000)
    with pytest.raises(ACError) as e:
        lay.synchronize()
    waited = time.perf_counter() - t0
    assert e.value.status == AC_ERR_TIMEOUT
    assert 0.019 <= waited < 1.5, waited
    lay.synchronize()  # the error word was cleared
    O1 = lay.forward(Q, K, V)
    lay.synchronize()
    assert torch.equal(O0, O1)
    lay.close()
