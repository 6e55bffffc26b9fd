"""The diagnostics harness (per-layer SQNR, per-tap relative std of Y, row-norm
balancing preset): closed forms on the CPU, agreement with the oracle's Y and SQNR
on the GPU."""
import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import diagnostics, synth, wino
from tests.gpu_util import to_device_input

P4, P6 = synth.POINTS_F4, synth.POINTS_F6


@pytest.mark.parametrize("m,pts", [(2, synth.POINTS_F2), (4, P4), (6, P6)])
def test_rownorm_scales_are_inverse_row_norms(m, pts):
    op = oracle.Plan(m, pts)
    sb, sg = diagnostics.rownorm_scales(m, pts)
    np.testing.assert_allclose(sb, 1.0 / np.linalg.norm(op.BT_d, axis=1), rtol=1e-6)
    np.testing.assert_allclose(sg, 1.0 / np.linalg.norm(op.G_d, axis=1), rtol=1e-6)


def test_per_tap_relative_std_closed_form():
    """Y[:, tap, :] = c_tap * Z: the std of tap k is |c_k| std(Z), relative to the mean |c|."""
    r = np.random.default_rng(3)
    n = 6
    c = r.uniform(0.1, 5.0, n * n) * r.choice([-1.0, 1.0], n * n)
    Z = r.standard_normal((40, 1, 24))
    Y = c[None, :, None] * Z
    rel = diagnostics.per_tap_relative_std(Y, n)
    np.testing.assert_allclose(rel.reshape(-1), np.abs(c) / np.abs(c).mean(), rtol=1e-12)


def test_sqnr_db_closed_form():
    ref = np.ones(100)
    assert abs(diagnostics.sqnr_db(ref, ref + 0.1) - 20.0) < 1e-9
    assert diagnostics.sqnr_db(ref, ref) == float("inf")


def _case(name):
    layer = synth.workload(name)[0]
    x_f32, x_bits = synth.make_input(layer)
    return layer, x_f32, x_bits, synth.make_weights(layer)


@pytest.mark.gpu
@pytest.mark.parametrize("y_groups", [wino.YGROUPS_TILE, wino.YGROUPS_TAP])
def test_diagnostics_match_the_oracle(cuda_dev, y_groups):
    layer, x_f32, x_bits, w = _case("tiny")
    sb, sg = diagnostics.rownorm_scales(layer.m, layer.points)
    d = diagnostics.diagnose(layer.m, layer.points, sb, sg, layer.group, to_device_input(x_f32, x_bits), w,
                             y_groups=y_groups)
    per_tap = y_groups == wino.YGROUPS_TAP
    ref = oracle.run_pipeline(oracle.Plan(layer.m, layer.points, sb, sg), x_f32, w, layer.group, per_tap=per_tap)
    assert np.array_equal(d["Y"], ref["Y"])
    assert np.array_equal(d["rel_std_Y"], diagnostics.per_tap_relative_std(ref["Y"], layer.n))
    s_orc = oracle.sqnr_db(oracle.conv_direct_f64(x_f32, w), ref["out"])
    assert abs(d["sqnr_db"] - s_orc) <= 0.01


@pytest.mark.gpu
@pytest.mark.parametrize("m", [4, 6])
def test_rownorm_preset_flattens_y_and_recovers_sqnr(cuda_dev, m):
    """The pages' diagnosis (Fig. 3): under the standard (identity) scales Y's per-tap
    spread is large and the tile-grouped output collapses; the balancing preset
    flattens the spread and recovers the SQNR."""
    layer = synth.random_layer(0, m, 1, 16, 16, 32, 32, 32, dtype="f32", act="normal", scales="identity",
                               w_var_num=1.0, workload="diag")
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    x = to_device_input(x_f32, x_bits)
    ident = diagnostics.diagnose(m, layer.points, None, None, 32, x, w)
    sb, sg = diagnostics.rownorm_scales(m, layer.points)
    bal = diagnostics.diagnose(m, layer.points, sb, sg, 32, x, w)
    assert ident["spread"] > 10.0 * bal["spread"]
    assert bal["sqnr_db"] > ident["sqnr_db"] + 20.0
