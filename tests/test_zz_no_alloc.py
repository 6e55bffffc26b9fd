"""GPU test of wino_conv2d_int8_noalloc, the entry point for callers that
cannot allocate device memory (no cudaMalloc available or permitted where
they run, or no way to hand a workspace through their interface).

The entry point runs the same convolution as wino_conv2d_int8 with its
scratch in the library's fixed device array instead of a caller workspace.
Both paths run the same kernels on the same inputs, so any difference would be
a stale-scratch or aliasing bug: the outputs are compared byte for byte.
Before the checked calls, a call of another shape and plan leaves different
contents in the array (Y absmax table, scales, error word), and the checked
shape is then called twice in a row through the C ABI.  A forced bounded-wait
expiry is read back through wino_check_device_error_noalloc.  This file is
collected last so that a run stopping at the first failure has already run
every other test.
"""
import numpy as np
import pytest
import torch

from group_wise_int8_b200 import synth, wino
from tests.gpu_util import to_device_input

pytestmark = pytest.mark.gpu

CASES = [
    # m, N, H, W, Cin, Cout, G, dtype, out dtype
    (6, 2, 13, 11, 64, 96, 32, "bf16", torch.float32),
    (4, 1, 16, 16, 32, 32, 32, "f32", torch.bfloat16),
]


def _setup(seed, case, debug=0, gemm=wino.GEMM_AUTO):
    m, N, H, W, Cin, Cout, G, dtype, out_dtype = case
    layer = synth.random_layer(seed, m, N, H, W, Cin, Cout, G, dtype=dtype,
                               act="relu_normal" if dtype == "bf16" else "normal", scales="loguniform",
                               workload="noalloc")
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    plan = wino.Plan(m, layer.points, sb, sg, G, debug=debug, gemm=gemm)
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    return plan, x, wt


def _call_noalloc(plan, x, wt, case):
    m, N, H, W, Cin, Cout, G, dtype, out_dtype = case
    y = torch.full((N, H, W, Cout), float("nan"), dtype=out_dtype, device="cuda")
    lib = wino.load_library()
    rc = lib.wino_conv2d_int8_noalloc(plan._h, x.data_ptr(), wino.BF16 if dtype == "bf16" else wino.F32,
                                      N, H, W, Cin, wt.data_ptr(), Cout, y.data_ptr(),
                                      wino.BF16 if out_dtype == torch.bfloat16 else wino.F32,
                                      torch.cuda.current_stream().cuda_stream)
    return rc, y


def _raw(t):
    return t.view(torch.int16 if t.element_size() == 2 else torch.int32)


@pytest.mark.parametrize("which", [0, 1], ids=["f6_bf16_ragged", "f4_f32_tiny"])
def test_noalloc_matches_workspace_entry_point(cuda_dev, which):
    case, other = CASES[which], CASES[1 - which]
    m, N, H, W, Cin, Cout, G, dtype, out_dtype = case
    plan, x, wt = _setup(3, case)
    assert 0 < plan.workspace_bytes(N, H, W, Cin, Cout) <= wino.NOALLOC_SCRATCH_BYTES
    y_ref = plan.conv2d(x, wt, Cout, out_dtype=out_dtype)
    torch.cuda.synchronize()

    # leave another shape's intermediates (and its Y absmax table) in the scratch array
    oplan, ox, owt = _setup(4, other)
    rc, _ = _call_noalloc(oplan, ox, owt, other)
    assert rc == wino.OK
    torch.cuda.synchronize()

    for call in range(2):
        rc, y = _call_noalloc(plan, x, wt, case)
        assert rc == wino.OK, (call, rc)
        torch.cuda.synchronize()
        assert plan.check_device_error_noalloc(N, H, W, Cin, Cout) == wino.OK
        assert torch.equal(_raw(y), _raw(y_ref)), "call %d differs from wino_conv2d_int8" % call


def test_noalloc_reports_a_bounded_wait_expiry(cuda_dev):
    """WINO_DEBUG_FORCE_TIMEOUT makes the GEMM's first wait expire (1 ms, no hang); the error
    word in the scratch array reports it, and the next normal call clears it."""
    case = CASES[0]
    m, N, H, W, Cin, Cout, G, dtype, out_dtype = case
    bad, x, wt = _setup(5, case, debug=wino.DEBUG_FORCE_TIMEOUT, gemm=wino.GEMM_TCGEN05)
    rc, _ = _call_noalloc(bad, x, wt, case)
    assert rc == wino.OK
    assert bad.check_device_error_noalloc(N, H, W, Cin, Cout) == wino.ERR_DEVICE_TIMEOUT
    good, x, wt = _setup(5, case, gemm=wino.GEMM_TCGEN05)
    rc, y = _call_noalloc(good, x, wt, case)
    assert rc == wino.OK
    assert good.check_device_error_noalloc(N, H, W, Cin, Cout) == wino.OK
    assert torch.equal(_raw(y), _raw(good.conv2d(x, wt, Cout, out_dtype=out_dtype)))


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_dev):
    plan = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    N, H, W, C = 128, 56, 56, 64
    assert plan.workspace_bytes(N, H, W, C, C) > wino.NOALLOC_SCRATCH_BYTES
    x = torch.zeros(16, dtype=torch.uint8, device="cuda")
    lib = wino.load_library()
    rc = lib.wino_conv2d_int8_noalloc(plan._h, x.data_ptr(), wino.BF16, N, H, W, C, x.data_ptr(), C,
                                      x.data_ptr(), wino.BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == wino.ERR_WORKSPACE
    assert plan.check_device_error_noalloc(N, H, W, C, C) == wino.ERR_WORKSPACE
