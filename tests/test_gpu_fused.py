"""GPU parity of the fused small-channel path (one kernel: input transform, both
GEMM passes of the recompute path and the output transform, with Vq and Yq
kept in shared memory) against the CPU oracle.

With the debug option the kernel also writes Vq, sV, Yq and sY to the
workspace in the staged layouts; every one of them, the transformed weights
and the output are compared bit for bit (fp32 outputs as values, bf16 outputs
as the bf16 of the oracle's fp32 output).  The cases cover F(2,3), F(4,3) and
F(6,3), G = 32 and 64, 32 and 64 channels, fp32 and bf16 input and output,
ragged images, a single pixel, a partial last unit of 16 tiles, and enough
tiles that CTAs take several units.  The same layers on the staged kernels
(the default) give the same output bytes.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth, wino
from tests.gpu_util import assert_bits_equal, bf16_round, rel_l2, run_gpu, run_oracle, to_device_input

pytestmark = pytest.mark.gpu

P2, P4, P6 = synth.POINTS_F2, synth.POINTS_F4, synth.POINTS_F6

# name: (m, points, N, H, W, Cin=Cout, G, dtype, act, scales)
CASES = {
    "f6_c64_g32_ragged": (6, P6, 2, 13, 11, 64, 32, "bf16", "relu_normal", "loguniform"),
    "f6_c64_g64_outliers": (6, P6, 1, 20, 20, 64, 64, "bf16", "student_t_outliers", "loguniform"),
    "f4_c64_g32": (4, P4, 2, 17, 19, 64, 32, "bf16", "relu_normal", "loguniform"),
    "f2_c64_g32_f32": (2, P2, 1, 15, 14, 64, 32, "f32", "normal", "loguniform"),
    "f6_c32_g32_f32": (6, P6, 1, 16, 16, 32, 32, "f32", "normal", "identity"),
    "f4_c32_g32": (4, P4, 3, 9, 10, 32, 32, "bf16", "normal", "loguniform"),
    "f6_one_pixel": (6, P6, 3, 1, 1, 64, 32, "bf16", "relu_normal", "identity"),
    "f6_many_units": (6, P6, 30, 56, 56, 64, 32, "bf16", "relu_normal", "loguniform"),   # 3000 tiles, 188 units
}


def _case(name):
    m, pts, N, H, W, C, G, dtype, act, scales = CASES[name]
    layer = synth.random_layer(21, m, N, H, W, C, C, G, dtype=dtype, act=act, scales=scales, w_var_num=2.0,
                               workload="fused_" + name)
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    return m, pts, G, x_f32, x_bits, w, sb, sg


_ref = {}


@pytest.mark.parametrize("out_dtype", [torch.float32, torch.bfloat16], ids=["f32_out", "bf16_out"])
@pytest.mark.parametrize("name", list(CASES))
def test_fused_path_bit_exact(cuda_dev, name, out_dtype):
    m, pts, G, x_f32, x_bits, w, sb, sg = _case(name)
    if name not in _ref:
        _ref[name] = run_oracle(m, pts, sb, sg, G, x_f32, w)
    ref = _ref[name]
    got = run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=out_dtype, debug=wino.DEBUG_YQ,
                  fused=wino.FUSED_ON)
    N, H, W, C = x_f32.shape
    assert got["plan"].resolved_variants(N, H, W, C, C) == wino.VARIANT_FUSED
    assert got["plan"].launches_per_call(N, H, W, C, C) == 1
    for k in ("Uq", "sU", "Vq", "sV", "Yq", "sY"):
        assert_bits_equal(k, got[k], ref[k])
    want = ref["out"] if out_dtype == torch.float32 else bf16_round(ref["out"])
    assert_bits_equal("out", got["out"], want)
    assert rel_l2(got["out"], want) <= 1e-5
    assert abs(oracle.sqnr_db(ref["ref"], got["out"]) - oracle.sqnr_db(ref["ref"], want)) <= 0.01


@pytest.mark.parametrize("name", ["f6_c64_g32_ragged", "f4_c32_g32", "f6_many_units"])
def test_fused_and_staged_paths_give_the_same_bytes(cuda_dev, name):
    m, pts, G, x_f32, x_bits, w, sb, sg = _case(name)
    N, H, W, C = x_f32.shape
    x = to_device_input(x_f32, x_bits)
    outs = []
    for fused in (wino.FUSED_ON, wino.FUSED_AUTO):
        plan = wino.Plan(m, pts, sb, sg, G, fused=fused)
        wt = plan.transform_weights(torch.from_numpy(w).cuda())
        ws = torch.full((plan.workspace_bytes(N, H, W, C, C),), 0x7f, dtype=torch.uint8, device="cuda")
        y = plan.conv2d(x, wt, C, out_dtype=torch.bfloat16, workspace=ws)
        torch.cuda.synchronize()
        assert plan.check_device_error(ws, N, H, W, C, C) == wino.OK
        assert bool(plan.resolved_variants(N, H, W, C, C) & wino.VARIANT_FUSED) == (fused == wino.FUSED_ON)
        outs.append(y.view(torch.int16).cpu())
    assert torch.equal(outs[0], outs[1])


def test_fused_path_without_debug_copies_has_a_small_workspace(cuda_dev):
    m, pts, G, x_f32, x_bits, w, sb, sg = _case("f6_c64_g32_ragged")
    N, H, W, C = x_f32.shape
    plan = wino.Plan(m, pts, sb, sg, G, fused=wino.FUSED_ON)
    staged = wino.Plan(m, pts, sb, sg, G)
    assert plan.workspace_bytes(N, H, W, C, C) <= 4096 < staged.workspace_bytes(N, H, W, C, C)
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.empty(plan.workspace_bytes(N, H, W, C, C), dtype=torch.uint8, device="cuda")
    y = plan.conv2d(x, wt, C, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    with pytest.raises(wino.WinoError) as e:
        plan.debug_dump(ws, N, H, W, C, C, wino.DUMP_VQ)
    assert e.value.status == wino.ERR_UNSUPPORTED
    ref = run_oracle(m, pts, sb, sg, G, x_f32, w)
    assert_bits_equal("out", y.cpu().numpy(), ref["out"])
