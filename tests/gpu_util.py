"""Helpers shared by the GPU parity tests: run one layer through the C ABI
(with the debug dumps) and through the CPU oracle on the same seeded bytes."""
import math

import numpy as np
import torch

import oracle
from group_wise_int8_b200 import synth, wino


def to_device_input(x_f32, x_bits):
    if x_bits is not None:
        return torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x_f32)).cuda()


def weight_dumps(plan, wt: torch.Tensor, Cin: int, Cout: int):
    """Split the transformed-weight buffer: Uq [n2][Cout][Cin], sU [n2][Cin/G][Cout]."""
    n2, G = plan.n * plan.n, plan.group
    raw = wt.cpu().numpy()
    uq_bytes = n2 * Cout * Cin
    off = (uq_bytes + 255) // 256 * 256
    Uq = raw[:uq_bytes].view(np.int8).reshape(n2, Cout, Cin)
    sU = raw[off:off + 4 * n2 * (Cin // G) * Cout].view(np.float32).reshape(n2, Cin // G, Cout)
    return Uq, np.ascontiguousarray(sU.transpose(0, 2, 1))


def run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=torch.float32, y_path=wino.YPATH_AUTO,
            gemm=wino.GEMM_AUTO, debug=0, y_groups=wino.YGROUPS_TILE, x_int8=False, int8_transforms=False,
            fused=wino.FUSED_AUTO):
    N, H, W, Cin = x_f32.shape
    Cout = w.shape[0]
    plan = wino.Plan(m, pts, sb, sg, G, y_path=y_path, gemm=gemm, debug=debug, y_groups=y_groups,
                     x_int8=x_int8, int8_transforms=int8_transforms, fused=fused)
    x = to_device_input(x_f32, x_bits)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device="cuda")
    out = plan.conv2d(x, wt, Cout, out_dtype=out_dtype, workspace=ws)
    torch.cuda.synchronize()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    res = {"out": out.float().cpu().numpy(), "plan": plan}
    res["Uq"], res["sU"] = weight_dumps(plan, wt, Cin, Cout)
    yp, gm = plan.resolved_config(N, H, W, Cin, Cout)
    res["y_path"], res["gemm"] = yp, gm
    # the fused path keeps Vq and Yq on chip: they exist only as its debug copies
    fused = bool(plan.resolved_variants(N, H, W, Cin, Cout) & wino.VARIANT_FUSED)
    if fused and not debug & wino.DEBUG_YQ:
        return res
    res["Vq"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_VQ)
    res["sV"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_SV)
    if debug & wino.DEBUG_YQ or yp == wino.YPATH_RECOMPUTE:
        res["Yq"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_YQ)
    if debug & wino.DEBUG_YQ:
        res["sY"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_SY)
    if yp == wino.YPATH_Y32:
        res["Y"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_Y32)
    if debug & wino.DEBUG_ACC32:
        res["acc"] = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_ACC32)
    return res


def run_oracle(m, pts, sb, sg, G, x_f32, w, want_acc=False, per_tap=False, x_int8=False, int8_transforms=False):
    res = oracle.run_pipeline(oracle.Plan(m, pts, sb, sg, int8_transforms=int8_transforms), x_f32, w, G,
                              want_acc=want_acc, per_tap=per_tap, x_int8=x_int8)
    res["ref"] = oracle.conv_direct_f64(x_f32, w)
    return res


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    nb = np.linalg.norm(b)
    return float(np.linalg.norm(a - b) / nb) if nb > 0 else float(np.linalg.norm(a - b))


def bf16_round(a):
    return synth.bf16_bits_to_f32(synth.f32_to_bf16_bits(np.asarray(a, np.float32)))


def assert_bits_equal(name, got, want):
    got = np.asarray(got)
    want = np.asarray(want)
    assert got.shape == want.shape, (name, got.shape, want.shape)
    if got.dtype.kind == "f":
        # +0 and -0 are the same code point for the quantiser; compare values, and NaN-free
        ok = np.array_equal(got, want)
    else:
        ok = np.array_equal(got, want)
    if not ok:
        diff = np.argwhere(got != want)
        first = tuple(diff[0])
        raise AssertionError("%s differs at %d of %d positions; first %s: got %r want %r"
                             % (name, len(diff), got.size, first, got[first], want[first]))
