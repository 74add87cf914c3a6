"""Calibration of N_max over a stack of layers (AdaCluster Sec. 4.1: k_max is
set so that the top 15% of layers -- the least compact, which need the most
clusters -- run full attention), host side: ac_calibrate_n_max on hand-worked
cases.  The GPU sweep over a synthetic layer stack is in
test_calibration_gpu.py."""
import pytest

from cluster_routed_sparse_b200 import _lib, api


def test_calibrate_picks_the_kth_largest_threshold():
    # units that fall back under N_max are those with fallback_at >= N_max
    f = [0, 96, 32, 160, 64, 0, 128, 32, 224, 64]
    assert api.calibrate_n_max(f, 0.15) == 160        # ceil(1.5) = 2 units: 224, 160
    assert sum(v >= 160 for v in f) == 2
    assert api.calibrate_n_max(f, 0.1) == 224         # 1 unit
    assert api.calibrate_n_max(f, 0.5) == 64          # 5 units: 224 160 128 96 64 (the tied 64 too: 6)
    assert api.calibrate_n_max(f, 0.0) == 225         # none
    assert api.calibrate_n_max(f, 1.0) == 32          # only the 8 multi-stage units can fall back


def test_calibrate_rejects_bad_input():
    with pytest.raises(_lib.ACError):
        api.calibrate_n_max([], 0.15)
    with pytest.raises(_lib.ACError):
        api.calibrate_n_max([5, 6], 1.5)
    with pytest.raises(_lib.ACError):
        api.calibrate_n_max([0, 0, 0], 0.5)           # single-stage units never fall back
