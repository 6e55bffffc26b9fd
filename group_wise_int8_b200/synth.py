"""Seeded synthetic layers for the group-wise int8 Winograd convolution.

This module only draws random numbers and describes layer shapes.  It holds
none of the method's arithmetic (no transform, no quantiser), so that the CPU
oracle and the CUDA path can both be fed from it without sharing any part of
the computation.

Stream discipline: every tensor comes from its own PCG64 stream, seeded with
the tuple (seed, workload id, layer index, tensor id).  Values are drawn in
fp64, cast to fp32, and rounded to bf16 (round-to-nearest-even on the fp32 bit
pattern) where the layer is bf16.

Workloads (the paper's models and datasets are not available, so these seeded
shapes and distributions stand in for them; the paper evaluates InstaFlow-0.9B,
SD v1.5 and ResNet-18/34 conv layers, "Data-Free Group-Wise Fully Quantized
Winograd Convolution via Learnable Scales", Sec. 5 setup):

  tiny        F(4,3), N1 C32 16x16, fp32 in/out, N(0,1) activations,
              w ~ N(0, 1/(9 Cin)), identity scales, points 0,+-1,+-2,inf, G=32.
  resnet18    F(6,3), N32 C64 56x56, bf16, ReLU(N(0,1)), w ~ N(0, 2/(9 Cin)),
              points 0,+-1,+-2,+-1/2,inf, log-uniform [0.5,2] scales, G=32.
  resnet34    F(6,3), batch 64, bf16: C64@56, C128@28, C256@14, C512@7.
  sd15        F(4,3) and F(6,3), batch 2, bf16, Student-t(3) activations with
              1% of channels scaled x20, w ~ N(0, 1/(9 Cin)), G=64:
              C320@64, C640@32, C1280@16, C1280@8.
  sd15_stack  the 44 3x3 ResNet-block convs of an SD-v1.5-shaped UNet, batch 8,
              F(6,3), G=64, activations as sd15.
"""
from __future__ import annotations

import dataclasses
import math
from typing import List, Optional, Sequence

import numpy as np

INF = math.inf

POINTS_F2 = (0.0, 1.0, -1.0, INF)
POINTS_F4 = (0.0, 1.0, -1.0, 2.0, -2.0, INF)
POINTS_F6 = (0.0, 1.0, -1.0, 2.0, -2.0, 0.5, -0.5, INF)

WORKLOAD_IDS = {"tiny": 0, "resnet18": 1, "resnet34": 2, "sd15": 3, "sd15_stack": 4, "probe": 5}

# tensor ids of the per-tensor streams
_T_X, _T_W, _T_SB, _T_SG, _T_OUTLIER = 1, 2, 3, 4, 5


@dataclasses.dataclass(frozen=True)
class Layer:
    """One 3x3, stride-1, pad-1 convolution layer of a workload."""
    workload: str
    index: int
    m: int
    N: int
    H: int
    W: int
    Cin: int
    Cout: int
    group: int
    dtype: str            # "f32" or "bf16" activations (and output in parity runs)
    act: str              # "normal", "relu_normal", "student_t_outliers"
    w_var_num: float      # weight variance = w_var_num / (9 Cin)
    scales: str           # "identity" or "loguniform"
    seed: int = 0

    @property
    def points(self):
        return {2: POINTS_F2, 4: POINTS_F4}.get(self.m, POINTS_F6)

    @property
    def n(self):
        return self.m + 2

    @property
    def tiles(self):
        return self.N * (-(-self.H // self.m)) * (-(-self.W // self.m))

    @property
    def direct_flops(self):
        """Direct-convolution-equivalent FLOPs: 2 N H W Cin Cout 9."""
        return 2.0 * self.N * self.H * self.W * self.Cin * self.Cout * 9

    def describe(self):
        return (f"F({self.m},3) N{self.N} Cin{self.Cin} Cout{self.Cout} {self.H}x{self.W} "
                f"G{self.group} {self.dtype}")


def _rng(seed: int, workload: str, layer: int, tensor: int) -> np.random.Generator:
    return np.random.default_rng([seed, WORKLOAD_IDS.get(workload, 99), layer, tensor])


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 bit patterns (uint16), round to nearest even. NaN-free input assumed."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = (u + 0x7FFF + ((u >> 16) & 1)) >> 16
    return rounded.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def make_input(layer: Layer):
    """Activation tensor, NHWC.

    Returns (x_f32, x_bf16_bits): x_f32 holds the exact values the convolution
    sees (for bf16 layers these are the bf16 values widened to fp32);
    x_bf16_bits is None for fp32 layers.
    """
    r = _rng(layer.seed, layer.workload, layer.index, _T_X)
    shape = (layer.N, layer.H, layer.W, layer.Cin)
    if layer.act == "normal":
        x = r.standard_normal(shape)
    elif layer.act == "relu_normal":
        x = np.maximum(r.standard_normal(shape), 0.0)
    elif layer.act == "student_t_outliers":
        x = r.standard_t(3.0, size=shape)
        k = max(1, int(round(0.01 * layer.Cin)))
        ro = _rng(layer.seed, layer.workload, layer.index, _T_OUTLIER)
        ch = ro.choice(layer.Cin, size=k, replace=False)
        x[..., ch] *= 20.0
    else:
        raise ValueError(layer.act)
    x32 = x.astype(np.float32)
    if layer.dtype == "bf16":
        bits = f32_to_bf16_bits(x32)
        return bf16_bits_to_f32(bits).reshape(shape), bits.reshape(shape)
    return np.ascontiguousarray(x32), None


def make_weights(layer: Layer) -> np.ndarray:
    """Weights [Cout][3][3][Cin] fp32, N(0, w_var_num / (9 Cin))."""
    r = _rng(layer.seed, layer.workload, layer.index, _T_W)
    std = math.sqrt(layer.w_var_num / (9.0 * layer.Cin))
    w = r.standard_normal((layer.Cout, 3, 3, layer.Cin)) * std
    return np.ascontiguousarray(w.astype(np.float32))


def make_scales(layer: Layer, shared_seed_layer: int = 0):
    """Diagonal scale vectors (S_B, S_G) as fp32 n-vectors, or (None, None) for identity.

    One scale set per network (the paper shares one learned set across all
    layers), so the stream is keyed on the workload, not the layer.
    """
    if layer.scales == "identity":
        return None, None
    n = layer.n
    rb = _rng(layer.seed, layer.workload, 1000 + layer.m, _T_SB)
    rg = _rng(layer.seed, layer.workload, 1000 + layer.m, _T_SG)
    lo, hi = math.log(0.5), math.log(2.0)
    sb = np.exp(rb.uniform(lo, hi, n)).astype(np.float32)
    sg = np.exp(rg.uniform(lo, hi, n)).astype(np.float32)
    return sb, sg


def random_layer(seed: int, m: int, N: int, H: int, W: int, Cin: int, Cout: int, group: int,
                 dtype: str = "bf16", act: str = "relu_normal", scales: str = "loguniform",
                 w_var_num: float = 2.0, workload: str = "custom") -> Layer:
    """A free-form layer for parity sweeps (ragged sizes, edge cases)."""
    return Layer(workload, seed, m, N, H, W, Cin, Cout, group, dtype, act, w_var_num, scales, seed)


def workload(name: str, seed: int = 0) -> List[Layer]:
    if name == "tiny":
        return [Layer("tiny", 0, 4, 1, 16, 16, 32, 32, 32, "f32", "normal", 1.0, "identity", seed)]
    if name == "resnet18":
        # [0] the F(6,3) layer; [1] the same layer as F(2,3) and [2] as F(4,3) (tile-size comparison)
        return [Layer("resnet18", i, m, 32, 56, 56, 64, 64, 32, "bf16", "relu_normal", 2.0, "loguniform", seed)
                for i, m in enumerate((6, 2, 4))]
    if name == "resnet34":
        shapes = [(64, 56), (128, 28), (256, 14), (512, 7)]
        return [Layer("resnet34", i, 6, 64, hw, hw, c, c, 32, "bf16", "relu_normal", 2.0,
                      "loguniform", seed) for i, (c, hw) in enumerate(shapes)]
    if name == "sd15":
        shapes = [(320, 64), (640, 32), (1280, 16), (1280, 8)]
        out = []
        for i, (c, hw) in enumerate(shapes):
            for j, m in enumerate((4, 6)):
                out.append(Layer("sd15", 2 * i + j, m, 2, hw, hw, c, c, 64, "bf16",
                                 "student_t_outliers", 1.0, "loguniform", seed))
        return out
    if name == "sd15_stack":
        # (Cin, Cout, resolution, count): 3x3 convs of the ResNet blocks of an
        # SD-v1.5-shaped UNet (320/640/1280/1280 channels, 2 blocks per down
        # level, 3 per up level, 2 in the mid block, concatenated skips).
        spec = [(320, 320, 64, 7), (640, 320, 64, 2), (960, 320, 64, 1),
                (320, 640, 32, 1), (640, 640, 32, 6), (960, 640, 32, 1), (1280, 640, 32, 1),
                (1920, 640, 32, 1),
                (640, 1280, 16, 1), (1280, 1280, 16, 6), (1920, 1280, 16, 1), (2560, 1280, 16, 2),
                (1280, 1280, 8, 11), (2560, 1280, 8, 3)]
        out = []
        for cin, cout, hw, cnt in spec:
            for _ in range(cnt):
                out.append(Layer("sd15_stack", len(out), 6, 8, hw, hw, cin, cout, 64, "bf16",
                                 "student_t_outliers", 1.0, "loguniform", seed))
        assert len(out) == 44
        return out
    if name == "probe":
        # Hadamard-stage capability probe: a compute-bound per-tap GEMM (T = 8192 tiles,
        # Cin = Cout = 2560, G = 64, F(6,3)) and a quarter-size copy (T = 2048) for profiling.
        return [Layer("probe", 0, 6, 2, 384, 384, 2560, 2560, 64, "bf16", "relu_normal", 2.0, "loguniform", seed),
                Layer("probe", 1, 6, 2, 192, 192, 2560, 2560, 64, "bf16", "relu_normal", 2.0, "loguniform", seed)]
    raise KeyError(name)
