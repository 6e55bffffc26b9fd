"""Stand-ins for a GPU memory checker (none is available where this library is
tested): the debug build and workspace guard bands.

* libwino_b200_debug.so is the library compiled with WINO_DEBUG: every kernel
  checks the element index of each global access against its buffer, skips an
  access that fails and records it in the device error word (no trap).
* The plan option WINO_DEBUG_GUARDS puts 4 KiB bands of a known byte before
  every workspace region and after the last; wino_check_guards reports the
  first band a call overwrote.

Every parity shape runs through the debug build with guard bands and the
stage dumps on both Y paths: no index check may fail, no band may change, and
every stage must still equal the CPU oracle's.  Two self-tests show that the
checks do fire: a byte written into a band from the host is reported with the
band's index, and the debug build's test hook (every checked element count one
less than its buffer) makes the kernels skip the last access of each buffer and
report WINO_ERR_DEVICE_BOUNDS -- the skipped output elements keep their old
contents, so nothing outside a buffer is ever touched.
"""
import numpy as np
import pytest
import torch

from group_wise_int8_b200 import synth, wino
from tests.gpu_util import assert_bits_equal, to_device_input, weight_dumps
from tests.test_gpu_parity import CASES, make_case, oracle_for

pytestmark = pytest.mark.gpu


def _run_debug(name, y_path, debug):
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
    N, H, W, Cin = x_f32.shape
    Cout = w.shape[0]
    plan = wino.Plan(m, pts, sb, sg, G, y_path=y_path, debug=debug, variant="debug")
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device="cuda")
    out = torch.full((N, H, W, Cout), float("nan"), dtype=torch.float32, device="cuda")
    plan.conv2d(x, wt, Cout, out=out, workspace=ws)
    torch.cuda.synchronize()
    return plan, wt, ws, out, (N, H, W, Cin, Cout)


@pytest.mark.parametrize("y_path", [wino.YPATH_RECOMPUTE, wino.YPATH_Y32])
@pytest.mark.parametrize("name", list(CASES))
def test_debug_build_with_guard_bands(cuda_dev, name, y_path):
    plan, wt, ws, out, shape = _run_debug(name, y_path, wino.DEBUG_GUARDS | wino.DEBUG_YQ)
    assert plan.check_device_error(ws, *shape) == wino.OK
    assert plan.check_guards(ws, *shape) == (wino.OK, -1)
    ref = oracle_for(name)
    N, H, W, Cin, Cout = shape
    Uq, sU = weight_dumps(plan, wt, Cin, Cout)
    assert_bits_equal("Uq", Uq, ref["Uq"])
    assert_bits_equal("sU", sU, ref["sU"])
    for k, what in (("Vq", wino.DUMP_VQ), ("sV", wino.DUMP_SV), ("Yq", wino.DUMP_YQ), ("sY", wino.DUMP_SY)):
        assert_bits_equal(k, plan.debug_dump(ws, *shape, what), ref[k])
    assert_bits_equal("out", out.cpu().numpy(), ref["out"])


def test_guard_check_reports_an_overwritten_band(cuda_dev):
    plan, wt, ws, out, shape = _run_debug("ragged_f6_cout96", wino.YPATH_AUTO, wino.DEBUG_GUARDS)
    assert plan.check_guards(ws, *shape) == (wino.OK, -1)
    ws[0] = 0                                   # the band in front of the first region
    assert plan.check_guards(ws, *shape) == (wino.ERR_GUARD, 0)
    ws[0] = 0xA5
    assert plan.check_guards(ws, *shape) == (wino.OK, -1)
    ws[plan.workspace_bytes(*shape) - 1] = 0x5A    # the band behind the last region
    rc, bad = plan.check_guards(ws, *shape)
    assert rc == wino.ERR_GUARD and bad > 0


def test_debug_build_index_checks_fire_and_skip(cuda_dev):
    plan, wt, ws, out, shape = _run_debug("ragged_f6_cout96", wino.YPATH_Y32, wino.DEBUG_SHRINK_BOUNDS)
    assert plan.check_device_error(ws, *shape) == wino.ERR_DEVICE_BOUNDS
    o = out.cpu().numpy().reshape(-1)
    assert np.isnan(o[-2:]).all()               # the last output pair failed its check and was skipped
    assert np.isfinite(o[:-2]).sum() > 0
    # the release build has no checks: the same hook changes nothing there
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case("ragged_f6_cout96")
    rel = wino.Plan(m, pts, sb, sg, G, y_path=wino.YPATH_Y32, debug=wino.DEBUG_SHRINK_BOUNDS)
    x = to_device_input(x_f32, x_bits)
    wt2 = rel.transform_weights(torch.from_numpy(w).cuda())
    ws2 = torch.empty(rel.workspace_bytes(*shape), dtype=torch.uint8, device="cuda")
    y = rel.conv2d(x, wt2, shape[-1], out_dtype=torch.float32, workspace=ws2)
    torch.cuda.synchronize()
    assert rel.check_device_error(ws2, *shape) == wino.OK
    assert_bits_equal("out", y.cpu().numpy(), oracle_for("ragged_f6_cout96")["out"])
