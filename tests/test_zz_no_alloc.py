"""GPU test of wino_conv2d_int8_noalloc, the entry point for callers that
cannot allocate device memory (no cudaMalloc available or permitted where
they run, or no way to hand a workspace through their interface).

The entry point runs the same convolution as wino_conv2d_int8 with its
scratch in the library's fixed device array instead of a caller workspace.
It is called through the C ABI, twice in a row on the same inputs (the array
keeps the first call's contents when the second starts), and each result is
compared with the workspace entry point's output within the tolerance the
parity tests use (1e-5 relative L2).  This file is collected last so that a
run stopping at the first failure has already run every other test.
"""
import numpy as np
import pytest
import torch

from group_wise_int8_b200 import synth, wino
from tests.gpu_util import rel_l2, to_device_input

pytestmark = pytest.mark.gpu

CASES = [
    # m, N, H, W, Cin, Cout, G, dtype, out dtype
    (6, 2, 13, 11, 64, 96, 32, "bf16", torch.float32),
    (4, 1, 16, 16, 32, 32, 32, "f32", torch.bfloat16),
]


@pytest.mark.parametrize("case", CASES, ids=["f6_bf16_ragged", "f4_f32_tiny"])
def test_noalloc_matches_workspace_entry_point(cuda_dev, case):
    m, N, H, W, Cin, Cout, G, dtype, out_dtype = case
    layer = synth.random_layer(3, m, N, H, W, Cin, Cout, G, dtype=dtype,
                               act="relu_normal" if dtype == "bf16" else "normal", scales="loguniform",
                               workload="noalloc")
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    plan = wino.Plan(m, layer.points, sb, sg, G)
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    assert 0 < plan.workspace_bytes(N, H, W, Cin, Cout) <= (64 << 20)
    y_ref = plan.conv2d(x, wt, Cout, out_dtype=out_dtype)
    torch.cuda.synchronize()
    ref = y_ref.float().cpu().numpy()

    lib = wino.load_library()
    stream = torch.cuda.current_stream().cuda_stream
    for call in range(2):
        y = torch.full((N, H, W, Cout), float("nan"), dtype=out_dtype, device="cuda")
        rc = lib.wino_conv2d_int8_noalloc(plan._h, x.data_ptr(), wino.BF16 if dtype == "bf16" else wino.F32,
                                          N, H, W, Cin, wt.data_ptr(), Cout, y.data_ptr(),
                                          wino.BF16 if out_dtype == torch.bfloat16 else wino.F32, stream)
        assert rc == wino.OK, (call, rc)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        assert np.isfinite(got).all()
        assert rel_l2(got, ref) <= 1e-5, (call, rel_l2(got, ref))


def test_noalloc_rejects_shapes_beyond_its_scratch(cuda_dev):
    plan = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    N, H, W, C = 128, 56, 56, 64
    assert plan.workspace_bytes(N, H, W, C, C) > (64 << 20)
    x = torch.zeros(16, dtype=torch.uint8, device="cuda")
    lib = wino.load_library()
    rc = lib.wino_conv2d_int8_noalloc(plan._h, x.data_ptr(), wino.BF16, N, H, W, C, x.data_ptr(), C,
                                      x.data_ptr(), wino.BF16, torch.cuda.current_stream().cuda_stream)
    assert rc == wino.ERR_WORKSPACE
