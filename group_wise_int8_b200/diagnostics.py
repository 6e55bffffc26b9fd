"""Diagnostics of the group-wise fully quantized Winograd layer ("Data-Free
Group-Wise Fully Quantized Winograd Convolution via Learnable Scales").

* `sqnr_db` -- the per-layer signal-to-quantisation-noise ratio the method's
  scale objective (Eq. 17) is stated in: 10 log10(sum ref^2 / sum (out - ref)^2)
  over the whole layer output, with `ref` the full-precision convolution.
* `per_tap_relative_std` -- Fig. 3 (a): the standard deviation of the
  Winograd-domain output Y at each tap, over all tiles and output channels,
  relative to the mean of those standard deviations over the taps (an n x n
  grid; the pages show its cross-shaped imbalance under standard scales).
* `rownorm_scales` -- the balancing preset: S_B[i] = 1/||B^T row i||,
  S_G[i] = 1/||G row i||, computed from the unscaled transforms.  For i.i.d.
  inputs and weights E[Y_ij^2] is proportional to the product of the row norms
  of B^T and G at points i and j, so this preset equalises the per-tap RMS of Y.
* `diagnose` -- one layer through the library with the fp32-Y path and the
  debug dumps, returning the SQNR against a float64 cuDNN convolution, the
  per-tap relative std of Y and of the requantised Yd, and the spread of the
  former (largest over smallest).

Run as a module for a table:  python -m group_wise_int8_b200.diagnostics
"""
from __future__ import annotations

import argparse
import math
from typing import Dict, Optional, Sequence

import numpy as np
import torch

from . import synth, wino


def sqnr_db(ref, out) -> float:
    ref = np.asarray(ref, np.float64)
    err = np.asarray(out, np.float64) - ref
    num, den = float(np.sum(ref * ref)), float(np.sum(err * err))
    return math.inf if den == 0.0 else 10.0 * math.log10(num / den)


def per_tap_relative_std(Y: np.ndarray, n: int) -> np.ndarray:
    """Y [T][n*n][Cout] -> [n][n]: std of each tap over (tiles, couts) / mean over taps."""
    Y = np.asarray(Y, np.float64)
    std = Y.transpose(1, 0, 2).reshape(n * n, -1).std(axis=1)
    mean = std.mean()
    return (std / mean if mean > 0 else std).reshape(n, n)


def rownorm_scales(m: int, points: Sequence[float]):
    """(S_B, S_G) = (1/||B^T_i||, 1/||G_i||) of the unscaled transforms, fp32."""
    BT, G, _ = wino.Plan(m, points, None, None, 32).matrices()
    sb = 1.0 / np.linalg.norm(np.asarray(BT, np.float64), axis=1)
    sg = 1.0 / np.linalg.norm(np.asarray(G, np.float64), axis=1)
    return sb.astype(np.float32), sg.astype(np.float32)


def reference_conv_f64(x: torch.Tensor, w: np.ndarray) -> np.ndarray:
    """Full-precision 3x3 stride-1 pad-1 correlation in float64 (cuDNN), NHWC out."""
    xt = x.to(torch.float64).permute(0, 3, 1, 2)
    wt = torch.from_numpy(np.asarray(w, np.float64)).to(x.device).permute(0, 3, 1, 2)
    return torch.nn.functional.conv2d(xt, wt, padding=1).permute(0, 2, 3, 1).cpu().numpy()


def diagnose(m: int, points: Sequence[float], S_B, S_G, G: int, x: torch.Tensor, w: np.ndarray,
             y_groups: int = wino.YGROUPS_TILE, gemm: int = wino.GEMM_AUTO, x_int8: bool = False,
             int8_transforms: bool = False) -> Dict[str, object]:
    """x: device NHWC (bf16 or fp32), w: host [Cout][3][3][Cin] fp32.  x_int8 / int8_transforms:
    the alternative readings of the input side (int8 x per pixel group, int8 B^T and A^T)."""
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    n = m + 2
    plan = wino.Plan(m, points, S_B, S_G, G, y_path=wino.YPATH_Y32, gemm=gemm, debug=wino.DEBUG_YQ,
                     y_groups=y_groups, x_int8=x_int8, int8_transforms=int8_transforms)
    wt = plan.transform_weights(torch.from_numpy(np.ascontiguousarray(w, np.float32)).to(x.device))
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout), dtype=torch.uint8, device=x.device)
    out = plan.conv2d(x, wt, Cout, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    Y = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_Y32)
    Yq = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_YQ).astype(np.float64)
    sY = plan.debug_dump(ws, N, H, W, Cin, Cout, wino.DUMP_SY).astype(np.float64)
    T = Y.shape[0]
    if y_groups == wino.YGROUPS_TAP:
        Yd = Yq * np.repeat(sY, G, axis=2)
    else:
        Yd = Yq * np.repeat(sY, G, axis=1)[:, None, :]
    rel = per_tap_relative_std(Y, n)
    ref = reference_conv_f64(x, w)
    return {
        "sqnr_db": sqnr_db(ref, out.cpu().numpy()),
        "rel_std_Y": rel,
        "rel_std_Yd": per_tap_relative_std(Yd.reshape(T, n * n, Cout), n),
        "spread": float(rel.max() / rel.min()) if rel.min() > 0 else math.inf,
        "out": out, "Y": Y,
    }


def _layer_inputs(layer: synth.Layer, dev: str):
    x_f32, x_bits = synth.make_input(layer)
    if x_bits is not None:
        x = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).to(dev)
    else:
        x = torch.from_numpy(x_f32).to(dev)
    return x, synth.make_weights(layer)


def main(argv: Optional[Sequence[str]] = None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--workload", default="resnet18", help="workload[:layer] from synth.workload")
    ap.add_argument("--m", type=int, default=0, help="override the tile size m (2, 4 or 6)")
    args = ap.parse_args(argv)
    name, _, idx = args.workload.partition(":")
    layer = synth.workload(name)[int(idx or 0)]
    if args.m:
        layer = synth.random_layer(layer.seed, args.m, layer.N, layer.H, layer.W, layer.Cin, layer.Cout,
                                   layer.group, layer.dtype, layer.act, layer.scales, layer.w_var_num, layer.workload)
    x, w = _layer_inputs(layer, "cuda")
    sb_l, sg_l = synth.make_scales(layer)
    presets = {"identity": (None, None), "rownorm": rownorm_scales(layer.m, layer.points),
               "layer scales": (sb_l, sg_l)}
    print("layer:", layer.describe())
    for yg, yname in ((wino.YGROUPS_TILE, "tile groups"), (wino.YGROUPS_TAP, "per-tap groups")):
        for pname, (sb, sg) in presets.items():
            d = diagnose(layer.m, layer.points, sb, sg, layer.group, x, w, y_groups=yg)
            print("%-15s %-13s SQNR %7.2f dB   per-tap std of Y: max/min %8.1f" % (yname, pname, d["sqnr_db"],
                                                                                     d["spread"]))
            if yg == wino.YGROUPS_TILE:
                for row in d["rel_std_Y"]:
                    print("      " + " ".join("%6.2f" % v for v in row))
    sb, sg = presets["rownorm"]
    for xi, it in ((True, False), (False, True), (True, True)):
        d = diagnose(layer.m, layer.points, sb, sg, layer.group, x, w, x_int8=xi, int8_transforms=it)
        print("tile groups     rownorm       SQNR %7.2f dB   x_int8=%d int8_transforms=%d"
              % (d["sqnr_db"], xi, it))


if __name__ == "__main__":
    main()
