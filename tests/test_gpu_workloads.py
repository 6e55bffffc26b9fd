"""Full-size sampled parity on every configured layer.

The GPU runs the whole layer in the launch configuration the benchmark times
(default options: automatic Y path, tcgen05 GEMM, bf16 output).  Every output
pixel of image i depends only on image i and the weights, so the CPU oracle
recomputes sampled images one at a time.  For those images the quantised input
transform (Vq, sV) and the GEMM's result on the layer's Y path (int8 Yq on the
recompute path, fp32 Y on the fp32-Y path) are compared bit for bit with the
oracle's tiles, and the bf16 output element by element (equal to the bf16 of
the oracle's fp32 output; the relative L2 and the SQNR to 0.01 dB are kept as
secondary checks).  The transformed weights are compared in full, bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth, wino
from tests.gpu_util import assert_bits_equal, bf16_round, rel_l2, to_device_input, weight_dumps

pytestmark = pytest.mark.gpu


def _layers():
    out = []
    for name in ("resnet18", "resnet34", "sd15"):
        for layer in synth.workload(name):
            out.append(layer)
    seen = set()
    for layer in synth.workload("sd15_stack"):
        key = (layer.Cin, layer.Cout, layer.H)
        if key not in seen:
            seen.add(key)
            out.append(layer)
    return out


LAYERS = _layers()


@pytest.mark.parametrize("layer", LAYERS, ids=[f"{l.workload}{l.index}-{l.describe().replace(' ', '_')}" for l in LAYERS])
def test_full_size_layer_sampled(cuda_dev, layer):
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    plan = wino.Plan(layer.m, layer.points, sb, sg, layer.group)
    N, H, W, Cin, Cout = layer.N, layer.H, layer.W, layer.Cin, layer.Cout
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device="cuda")
    y = plan.conv2d(x, wt, Cout, out_dtype=torch.bfloat16, workspace=ws)
    torch.cuda.synchronize()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    y = y.float().cpu().numpy()
    y_path, _ = plan.resolved_config(N, H, W, Cin, Cout)
    gVq = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_VQ)
    gsV = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_SV)
    gY = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_YQ if y_path == wino.YPATH_RECOMPUTE else wino.DUMP_Y32)

    op = oracle.Plan(layer.m, layer.points, sb, sg)
    Uq, sU, _ = oracle.weight_transform(op, w, layer.group)
    gUq, gsU = weight_dumps(plan, wt, Cin, Cout)
    assert_bits_equal("Uq", gUq, Uq)
    assert_bits_equal("sU", gsU, sU)
    tpi = -(-H // layer.m) * -(-W // layer.m)           # tiles per image
    images = [0, N - 1] if layer.workload != "sd15_stack" else [N - 1]
    for i in sorted(set(images)):
        xi = np.ascontiguousarray(x_f32[i:i + 1])
        res = oracle.run_pipeline(op, xi, w, layer.group)
        tiles = slice(i * tpi, (i + 1) * tpi)
        assert_bits_equal("Vq[image %d]" % i, gVq[tiles], res["Vq"])
        assert_bits_equal("sV[image %d]" % i, gsV[tiles], res["sV"])
        if y_path == wino.YPATH_RECOMPUTE:
            assert_bits_equal("Yq[image %d]" % i, gY[tiles], res["Yq"])
        else:
            assert_bits_equal("Y[image %d]" % i, gY[tiles], res["Y"])
        want = bf16_round(res["out"])
        got = y[i:i + 1]
        assert_bits_equal("out[image %d]" % i, got, want)
        assert rel_l2(got, want) <= 1e-5, (i, rel_l2(got, want))
        ref = oracle.conv_direct_f64(xi, w)
        assert abs(oracle.sqnr_db(ref, got) - oracle.sqnr_db(ref, want)) <= 0.01
