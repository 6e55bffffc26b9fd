"""ctypes wrapper around the C++ oracle (oracle/wino_oracle.cpp).

TEST INFRASTRUCTURE ONLY.  Each function calls one oracle stage; the Python
side only allocates arrays and passes pointers.  `run_pipeline` chains the
stages in the order the method applies them (weight transform, input
transform, Hadamard product, Y requantisation, output transform).
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Dict, Optional, Sequence

import numpy as np

from . import build as _build

_lib = None

_f32p = ctypes.POINTER(ctypes.c_float)
_f64p = ctypes.POINTER(ctypes.c_double)
_i8p = ctypes.POINTER(ctypes.c_int8)
_i32p = ctypes.POINTER(ctypes.c_int32)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.orc_set_threads.argtypes = [ctypes.c_int]
        L.orc_set_threads.restype = ctypes.c_int
        L.orc_plan.argtypes = [ctypes.c_int, _f64p, _f32p, _f32p, _f64p, _f32p, _f64p, _f64p, _f32p]
        L.orc_plan.restype = ctypes.c_int
        L.orc_quantize.argtypes = [_f32p, ctypes.c_int, _i8p, _f32p]
        L.orc_quantize.restype = None
        L.orc_quantize_matrix.argtypes = [_f32p, ctypes.c_int]
        L.orc_quantize_matrix.restype = None
        L.orc_quantize_input.argtypes = [_f32p, ctypes.c_long, ctypes.c_int, ctypes.c_int, _f32p]
        L.orc_quantize_input.restype = ctypes.c_int
        L.orc_weight_transform.argtypes = [ctypes.c_int, _f64p, _f32p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, _f32p, _i8p, _f32p]
        L.orc_input_transform.argtypes = [ctypes.c_int, _f32p, _f32p, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p, _i8p, _f32p]
        L.orc_hadamard.argtypes = [ctypes.c_int, _i8p, _f32p, _i8p, _f32p, ctypes.c_long, ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, _f32p, _i32p]
        L.orc_y_requant.argtypes = [ctypes.c_int, _f32p, ctypes.c_long, ctypes.c_int, ctypes.c_int, _i8p, _f32p]
        L.orc_output_transform.argtypes = [ctypes.c_int, _f32p, _i8p, _f32p, ctypes.c_int, ctypes.c_int,
                                           ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p]
        L.orc_y_requant_tap.argtypes = L.orc_y_requant.argtypes
        L.orc_output_transform_tap.argtypes = L.orc_output_transform.argtypes
        L.orc_conv_direct_f64.argtypes = [_f32p, _f32p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                          ctypes.c_int, ctypes.c_int, _f64p]
        L.orc_conv_wino_f64.argtypes = [ctypes.c_int, _f64p, _f64p, _f64p, _f32p, _f32p, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f64p]
        L.orc_conv_wino_f32.argtypes = [ctypes.c_int, _f32p, _f64p, _f32p, _f32p, _f32p, ctypes.c_int,
                                        ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, _f32p]
        for name in ("orc_weight_transform", "orc_input_transform", "orc_hadamard", "orc_y_requant",
                     "orc_output_transform", "orc_y_requant_tap", "orc_output_transform_tap",
                     "orc_conv_direct_f64", "orc_conv_wino_f64", "orc_conv_wino_f32"):
            getattr(L, name).restype = ctypes.c_int
        _lib = L
    return _lib


def _p(a: Optional[np.ndarray], t):
    if a is None:
        return ctypes.cast(None, t)
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(t)


def set_threads(t: int) -> int:
    """Number of OpenMP threads the oracle uses (0 = library default). Returns the count in use."""
    return lib().orc_set_threads(int(t))


class Plan:
    """Transform matrices of F(m,3) (see orc_plan).  int8_transforms: the alternative reading
    in which the fp32 B^T and A^T are each held as int8 with one scale (orc_quantize_matrix)."""

    def __init__(self, m: int, points: Sequence[float], S_B=None, S_G=None, int8_transforms: bool = False):
        n = m + 2
        self.m, self.n = m, n
        pts = np.ascontiguousarray(np.array(points, dtype=np.float64))
        assert pts.shape == (n,)
        sb = None if S_B is None else np.ascontiguousarray(np.asarray(S_B, dtype=np.float32))
        sg = None if S_G is None else np.ascontiguousarray(np.asarray(S_G, dtype=np.float32))
        self.BT_d = np.zeros((n, n), np.float64)
        self.BT_f = np.zeros((n, n), np.float32)
        self.G_d = np.zeros((n, 3), np.float64)
        self.AT_d = np.zeros((m, n), np.float64)
        self.AT_f = np.zeros((m, n), np.float32)
        rc = lib().orc_plan(m, _p(pts, _f64p), _p(sb, _f32p), _p(sg, _f32p), _p(self.BT_d, _f64p),
                            _p(self.BT_f, _f32p), _p(self.G_d, _f64p), _p(self.AT_d, _f64p),
                            _p(self.AT_f, _f32p))
        if rc != 0:
            raise ValueError("orc_plan failed: %d" % rc)
        if int8_transforms:
            lib().orc_quantize_matrix(_p(self.BT_f, _f32p), n * n)
            lib().orc_quantize_matrix(_p(self.AT_f, _f32p), m * n)


def quantize(v: np.ndarray):
    v = np.ascontiguousarray(v, dtype=np.float32)
    q = np.zeros(v.shape, np.int8)
    s = np.zeros(1, np.float32)
    lib().orc_quantize(_p(v, _f32p), v.size, _p(q, _i8p), _p(s, _f32p))
    return q, float(s[0])


def quantize_input(x: np.ndarray, G: int) -> np.ndarray:
    """x [..., C] with each pixel's G consecutive channels through Q, returned as s * q (fp32)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    C = x.shape[-1]
    xq = np.zeros_like(x)
    rc = lib().orc_quantize_input(_p(x, _f32p), x.size // C, C, G, _p(xq, _f32p))
    assert rc == 0
    return xq


def weight_transform(plan: Plan, w: np.ndarray, G: int, want_float: bool = False):
    Cout, _, _, Cin = w.shape
    n2 = plan.n * plan.n
    w = np.ascontiguousarray(w, dtype=np.float32)
    Uf = np.zeros((n2, Cout, Cin), np.float32) if want_float else None
    Uq = np.zeros((n2, Cout, Cin), np.int8)
    sU = np.zeros((n2, Cout, Cin // G), np.float32)
    rc = lib().orc_weight_transform(plan.m, _p(plan.G_d, _f64p), _p(w, _f32p), Cin, Cout, G,
                                    _p(Uf, _f32p), _p(Uq, _i8p), _p(sU, _f32p))
    assert rc == 0
    return Uq, sU, Uf


def input_transform(plan: Plan, x: np.ndarray, G: int, want_float: bool = False, quantize: bool = True):
    N, H, W, Cin = x.shape
    m, n2 = plan.m, plan.n * plan.n
    T = N * (-(-H // m)) * (-(-W // m))
    x = np.ascontiguousarray(x, dtype=np.float32)
    Vf = np.zeros((T, n2, Cin), np.float32) if want_float else None
    Vq = np.zeros((T, n2, Cin), np.int8) if quantize else None
    sV = np.zeros((T, n2, Cin // G), np.float32) if quantize else None
    rc = lib().orc_input_transform(m, _p(plan.BT_f, _f32p), _p(x, _f32p), N, H, W, Cin, G, _p(Vf, _f32p),
                                   _p(Vq, _i8p), _p(sV, _f32p))
    assert rc == 0
    return Vq, sV, Vf


def hadamard(n2: int, Vq, sV, Uq, sU, G: int, want_acc: bool = False):
    T, _, Cin = Vq.shape
    Cout = Uq.shape[1]
    Y = np.zeros((T, n2, Cout), np.float32)
    acc = np.zeros((n2, T, Cout, Cin // G), np.int32) if want_acc else None
    rc = lib().orc_hadamard(n2, _p(Vq, _i8p), _p(sV, _f32p), _p(Uq, _i8p), _p(sU, _f32p), T, Cin, Cout, G,
                            _p(Y, _f32p), _p(acc, _i32p))
    assert rc == 0
    return Y, acc


def y_requant(n2: int, Y: np.ndarray, G: int, per_tap: bool = False):
    """Y groups of G couts spanning all n2 taps of a tile (sY [T][Cout/G]), or, with
    per_tap (the Y_TAP reading), one group per tap (sY [T][n2][Cout/G])."""
    T, _, Cout = Y.shape
    Yq = np.zeros(Y.shape, np.int8)
    sY = np.zeros((T, n2, Cout // G) if per_tap else (T, Cout // G), np.float32)
    fn = lib().orc_y_requant_tap if per_tap else lib().orc_y_requant
    rc = fn(n2, _p(np.ascontiguousarray(Y), _f32p), T, Cout, G, _p(Yq, _i8p), _p(sY, _f32p))
    assert rc == 0
    return Yq, sY


def output_transform(plan: Plan, Yq, sY, N: int, H: int, W: int, G: int, per_tap: bool = False):
    Cout = Yq.shape[2]
    out = np.zeros((N, H, W, Cout), np.float32)
    fn = lib().orc_output_transform_tap if per_tap else lib().orc_output_transform
    rc = fn(plan.m, _p(plan.AT_f, _f32p), _p(Yq, _i8p), _p(np.ascontiguousarray(sY), _f32p), N, H, W, Cout,
            G, _p(out, _f32p))
    assert rc == 0
    return out


def conv_direct_f64(x: np.ndarray, w: np.ndarray) -> np.ndarray:
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    out = np.zeros((N, H, W, Cout), np.float64)
    rc = lib().orc_conv_direct_f64(_p(np.ascontiguousarray(x, np.float32), _f32p),
                                   _p(np.ascontiguousarray(w, np.float32), _f32p), N, H, W, Cin, Cout,
                                   _p(out, _f64p))
    assert rc == 0
    return out


def conv_wino_f64(plan: Plan, x: np.ndarray, w: np.ndarray) -> np.ndarray:
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    out = np.zeros((N, H, W, Cout), np.float64)
    rc = lib().orc_conv_wino_f64(plan.m, _p(plan.BT_d, _f64p), _p(plan.G_d, _f64p), _p(plan.AT_d, _f64p),
                                 _p(np.ascontiguousarray(x, np.float32), _f32p),
                                 _p(np.ascontiguousarray(w, np.float32), _f32p), N, H, W, Cin, Cout,
                                 _p(out, _f64p))
    assert rc == 0
    return out


def conv_wino_f32(plan: Plan, x: np.ndarray, w: np.ndarray) -> np.ndarray:
    N, H, W, Cin = x.shape
    Cout = w.shape[0]
    out = np.zeros((N, H, W, Cout), np.float32)
    rc = lib().orc_conv_wino_f32(plan.m, _p(plan.BT_f, _f32p), _p(plan.G_d, _f64p), _p(plan.AT_f, _f32p),
                                 _p(np.ascontiguousarray(x, np.float32), _f32p),
                                 _p(np.ascontiguousarray(w, np.float32), _f32p), N, H, W, Cin, Cout,
                                 _p(out, _f32p))
    assert rc == 0
    return out


def run_pipeline(plan: Plan, x: np.ndarray, w: np.ndarray, G: int, want_acc: bool = False,
                 per_tap: bool = False, x_int8: bool = False) -> Dict[str, np.ndarray]:
    """The full quantised pipeline, every stage kept for comparison (per_tap: the Y_TAP
    reading of the Y groups; x_int8: x itself group-quantised before the input transform)."""
    N, H, W, _ = x.shape
    n2 = plan.n * plan.n
    if x_int8:
        x = quantize_input(x, G)
    Uq, sU, _ = weight_transform(plan, w, G)
    Vq, sV, _ = input_transform(plan, x, G)
    Y, acc = hadamard(n2, Vq, sV, Uq, sU, G, want_acc=want_acc)
    Yq, sY = y_requant(n2, Y, G, per_tap)
    out = output_transform(plan, Yq, sY, N, H, W, G, per_tap)
    return dict(Uq=Uq, sU=sU, Vq=Vq, sV=sV, Y=Y, acc=acc, Yq=Yq, sY=sY, out=out)


def sqnr_db(ref: np.ndarray, out: np.ndarray) -> float:
    """10 log10(sum ref^2 / sum (out - ref)^2) over the whole layer output (fp64)."""
    ref = np.asarray(ref, np.float64)
    err = np.asarray(out, np.float64) - ref
    num, den = float(np.sum(ref * ref)), float(np.sum(err * err))
    if den == 0.0:
        return math.inf
    return 10.0 * math.log10(num / den)
