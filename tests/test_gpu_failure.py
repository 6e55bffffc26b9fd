"""Failure detection without a GPU fault: a bounded device wait that runs out.

The plan's WINO_DEBUG_FORCE_TIMEOUT hook makes the tcgen05 GEMM first wait 1 ms
on an mbarrier that nothing completes.  The wait expires, the CTA raises its
abort flag and the workspace's error word, every role drains its in-flight
TMA loads and MMAs, frees its TMEM and returns; the host then reads
WINO_ERR_DEVICE_TIMEOUT.  The context stays usable: the next normal call on
the same workspace succeeds and matches the oracle.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth, wino
from tests.gpu_util import rel_l2, to_device_input

pytestmark = pytest.mark.gpu


def test_bounded_wait_expiry_is_reported_and_recoverable(cuda_dev):
    layer = synth.random_layer(5, 6, 1, 12, 12, 64, 64, 32, workload="timeout")
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    N, H, W, Cin, Cout = layer.N, layer.H, layer.W, layer.Cin, layer.Cout
    x = to_device_input(x_f32, x_bits)
    wdev = torch.from_numpy(w).cuda()

    bad = wino.Plan(6, layer.points, sb, sg, 32, gemm=wino.GEMM_TCGEN05, debug=wino.DEBUG_FORCE_TIMEOUT)
    ws = torch.empty(bad.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device="cuda")
    wt = bad.transform_weights(wdev)
    bad.conv2d(x, wt, Cout, out_dtype=torch.float32, workspace=ws)
    assert bad.check_device_error(ws, N, H, W, Cin, Cout) == wino.ERR_DEVICE_TIMEOUT

    good = wino.Plan(6, layer.points, sb, sg, 32, gemm=wino.GEMM_TCGEN05)
    assert good.workspace_bytes(N, H, W, Cin, Cout) <= ws.numel()
    y = good.conv2d(x, good.transform_weights(wdev), Cout, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert good.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    ref = oracle.run_pipeline(oracle.Plan(6, layer.points, sb, sg), x_f32, w, 32)["out"]
    assert rel_l2(y.cpu().numpy(), ref) <= 1e-5
