"""The C-ABI library builds for sm_100a, loads, and exports every function
that include/ac.h declares; argument checks run without a GPU."""
import ctypes
import os
import re
import subprocess

import pytest

from conftest import ROOT
from cluster_routed_sparse_b200 import build, _lib

HEADER = os.path.join(ROOT, "include", "ac.h")


def _declared():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"^AC_API\s+[\w\s\*]+?\b(ac_\w+)\s*\(", txt, flags=re.M)))


def test_library_builds_and_exports_every_declared_symbol():
    path = build.build()
    lib = ctypes.CDLL(path)
    names = _declared()
    assert len(names) >= 14
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(_lib.SIGNATURES), set(names) ^ set(_lib.SIGNATURES)
    out = subprocess.run(["nm", "-D", "--defined-only", path], capture_output=True, text=True).stdout
    exported = set(re.findall(r" T (ac_\w+)", out))
    assert exported == set(names)


def test_config_struct_layout_matches_header(tmp_path):
    src = tmp_path / "s.c"
    src.write_text('#include <stdio.h>\n#include <stddef.h>\n#include "ac.h"\nint main(void){'
                   'printf("%zu %zu %zu %zu %zu\\n", sizeof(ac_config), offsetof(ac_config, seed),'
                   ' offsetof(ac_config, scale), sizeof(ac_stage_times), sizeof(ac_attn_counters));'
                   'return 0;}\n')
    exe = tmp_path / "s"
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), str(src), "-o", str(exe)], check=True)
    got = subprocess.run([str(exe)], capture_output=True, text=True).stdout.split()
    assert [int(x) for x in got] == [ctypes.sizeof(_lib.ACConfig), _lib.ACConfig.seed.offset,
                                     _lib.ACConfig.scale.offset, ctypes.sizeof(_lib.ACStageTimes),
                                     ctypes.sizeof(_lib.ACAttnCounters)]


def _create(**kw):
    lib = _lib.load()
    base = dict(Cq=16, m0=32, n_max=128, tau_mode=1, tau_value=0.5, topk=8, iters_q=10, iters_k=10,
                iters_warm=2, stage_rule=0, seed=1, scale=0.0, score_mode=0, tail_merge=0,
                unit0=0, compensate=0)
    dims = kw.pop("dims", (1, 2, 4096, 64))
    base.update(kw)
    cfg = _lib.ACConfig(**base)
    h = ctypes.c_void_p()
    return lib.ac_create(ctypes.byref(cfg), *dims, ctypes.byref(h)), h


@pytest.mark.parametrize("kw,expect", [
    (dict(Cq=0), _lib.AC_ERR_INVALID_ARG),
    (dict(Cq=5000), _lib.AC_ERR_INVALID_ARG),          # Cq > L
    (dict(m0=0), _lib.AC_ERR_INVALID_ARG),
    (dict(n_max=0), _lib.AC_ERR_INVALID_ARG),
    (dict(topk=0), _lib.AC_ERR_INVALID_ARG),
    (dict(tau_mode=7), _lib.AC_ERR_INVALID_ARG),
    (dict(tau_mode=2, tau_value=0.0), _lib.AC_ERR_INVALID_ARG),
    (dict(iters_k=-1), _lib.AC_ERR_INVALID_ARG),
    (dict(stage_rule=3), _lib.AC_ERR_INVALID_ARG),
    (dict(score_mode=2), _lib.AC_ERR_INVALID_ARG),
    (dict(tail_merge=3), _lib.AC_ERR_INVALID_ARG),
    (dict(unit0=-1), _lib.AC_ERR_INVALID_ARG),
    (dict(compensate=2), _lib.AC_ERR_INVALID_ARG),
    (dict(compensate=1, tail_merge=1), _lib.AC_ERR_INVALID_ARG),
    (dict(dims=(1, 2, 0, 64)), _lib.AC_ERR_INVALID_ARG),
    (dict(dims=(1, 2, 4096, 96)), _lib.AC_ERR_UNSUPPORTED),
])
def test_create_rejects_bad_arguments(kw, expect):
    st, h = _create(**kw)
    assert st == expect and not h.value


def test_null_arguments_rejected():
    lib = _lib.load()
    assert lib.ac_create(None, 1, 1, 1, 64, None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_destroy(None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_synchronize(None, None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_join(None, None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_layer_forward_host_async(None, None, None, None, None, 0, None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_check_wait_timeout(None, 1000, None) == _lib.AC_ERR_INVALID_ARG
    assert lib.ac_last_error_string(None) == b""


def test_create_without_gpu_reports_unsupported():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st, h = _create()
    assert st in (_lib.AC_ERR_UNSUPPORTED, _lib.AC_ERR_CUDA) and not h.value
