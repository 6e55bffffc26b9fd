"""Python binding of the C ABI in include/wino.h (argument marshalling only).

Every step of the convolution runs in the CUDA library libwino_b200.so; this
module only turns torch tensors into pointers and the current CUDA stream
into a handle, and raises on non-zero status codes.  There is no CPU path:
if the library is missing, loading fails with an error.
"""
from __future__ import annotations

import ctypes
import math
import os
from typing import Optional, Sequence

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libwino_b200.so")
# the same library compiled with WINO_DEBUG: index checks in every kernel (see include/wino.h)
LIB_PATH_DEBUG = os.path.join(HERE, "libwino_b200_debug.so")
LIB_PATHS = {"release": LIB_PATH, "debug": LIB_PATH_DEBUG}

OK = 0
ERR_INVALID_ARG = -1
ERR_UNSUPPORTED = -2
ERR_WORKSPACE = -3
ERR_CUDA = -4
ERR_DEVICE_TIMEOUT = -5
ERR_NOT_EXACT = -6
ERR_DEVICE_BOUNDS = -7
ERR_GUARD = -8

F32 = 0
BF16 = 1

YPATH_AUTO, YPATH_RECOMPUTE, YPATH_Y32 = 0, 1, 2
GEMM_AUTO, GEMM_TCGEN05, GEMM_SIMT = 0, 1, 2
DEBUG_YQ, DEBUG_ACC32, DEBUG_FORCE_TIMEOUT, DEBUG_GUARDS, DEBUG_SHRINK_BOUNDS = 1, 2, 4, 8, 16
YGROUPS_TILE, YGROUPS_TAP = 0, 1
VARIANT_SWAPPED_GEMM, VARIANT_SPLIT_INPUT, VARIANT_SPLIT_OUTPUT, VARIANT_FUSED, VARIANT_A_RESIDENT = 1, 2, 4, 8, 16
FUSED_AUTO, FUSED_OFF, FUSED_ON = 0, 1, 2
DUMP_VQ, DUMP_SV, DUMP_YQ, DUMP_SY, DUMP_Y32, DUMP_ACC32 = range(6)
NOALLOC_SCRATCH_BYTES = 64 << 20   # WINO_NOALLOC_SCRATCH_BYTES

EXPORTED = [
    "wino_plan", "wino_plan_destroy", "wino_plan_matrices", "wino_plan_info", "wino_weight_bytes",
    "wino_transform_weights", "wino_workspace_bytes", "wino_conv2d_int8", "wino_conv2d_int8_noalloc",
    "wino_check_device_error_noalloc", "wino_check_guards",
    "wino_host_staging_bytes",
    "wino_conv2d_int8_host", "wino_check_device_error", "wino_debug_dump", "wino_resolved_config",
    "wino_resolved_variants", "wino_launches_per_call", "wino_profile_begin", "wino_profile_end", "wino_last_cuda_error",
    "wino_status_string",
]


class WinoError(RuntimeError):
    def __init__(self, status: int, what: str, cuda: int = 0):
        super().__init__("%s failed: %s (%d)%s" % (what, _status_string(status), status,
                                                  (", cudaError %d" % cuda) if cuda else ""))
        self.status = status


class Opts(ctypes.Structure):
    _fields_ = [("y_path", ctypes.c_int), ("gemm", ctypes.c_int), ("debug", ctypes.c_int),
                ("y_groups", ctypes.c_int), ("x_int8", ctypes.c_int), ("int8_transforms", ctypes.c_int),
                ("fused", ctypes.c_int), ("reserved", ctypes.c_int)]


_libs = {}
_lib = None   # the release library once loaded
_vp = ctypes.c_void_p
_sz = ctypes.c_size_t
_i = ctypes.c_int


def load_library(path: Optional[str] = None, variant: str = "release"):
    """Load the CUDA library (raises OSError if it has not been built): the release build, or
    with variant="debug" the WINO_DEBUG build whose kernels check every index."""
    global _lib
    path = path or LIB_PATHS[variant]
    if path in _libs:
        return _libs[path]
    if not os.path.exists(path):
        raise OSError("CUDA library %s is missing: run `python -m group_wise_int8_b200.build`" % path)
    L = ctypes.CDLL(path)
    L.wino_plan.argtypes = [ctypes.POINTER(_vp), _i, ctypes.POINTER(ctypes.c_double), ctypes.POINTER(ctypes.c_float),
                            ctypes.POINTER(ctypes.c_float), _i, ctypes.POINTER(Opts)]
    L.wino_plan_destroy.argtypes = [_vp]
    L.wino_plan_matrices.argtypes = [_vp, ctypes.POINTER(ctypes.c_float), ctypes.POINTER(ctypes.c_double),
                                     ctypes.POINTER(ctypes.c_float)]
    L.wino_plan_info.argtypes = [_vp, ctypes.POINTER(_i), ctypes.POINTER(_i), ctypes.POINTER(_i)]
    L.wino_weight_bytes.argtypes = [_vp, _i, _i]
    L.wino_weight_bytes.restype = _sz
    L.wino_transform_weights.argtypes = [_vp, _vp, _i, _i, _vp, _sz, _vp]
    L.wino_workspace_bytes.argtypes = [_vp, _i, _i, _i, _i, _i]
    L.wino_workspace_bytes.restype = _sz
    L.wino_conv2d_int8.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _i, _vp, _sz, _vp]
    L.wino_conv2d_int8_noalloc.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _i, _vp]
    L.wino_check_device_error_noalloc.argtypes = [_vp, _i, _i, _i, _i, _i, _vp]
    L.wino_check_guards.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, ctypes.POINTER(_i)]
    L.wino_host_staging_bytes.argtypes = [_vp, _i, _i, _i, _i, _i, _i, _i]
    L.wino_host_staging_bytes.restype = _sz
    L.wino_conv2d_int8_host.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp, _i, _vp, _i, _vp, _sz, _vp]
    L.wino_check_device_error.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _vp]
    L.wino_debug_dump.argtypes = [_vp, _vp, _i, _i, _i, _i, _i, _i, _vp, _sz]
    L.wino_resolved_config.argtypes = [_vp, _i, _i, _i, _i, _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]
    L.wino_resolved_variants.argtypes = [_vp, _i, _i, _i, _i, _i, ctypes.POINTER(_i)]
    L.wino_launches_per_call.argtypes = [_vp, _i, _i, _i, _i, _i]
    L.wino_profile_begin.argtypes = [_vp, _i]
    L.wino_profile_end.argtypes = [_vp, ctypes.POINTER(ctypes.c_float), _i, ctypes.POINTER(_i), ctypes.POINTER(_i)]
    L.wino_last_cuda_error.argtypes = [_vp]
    L.wino_status_string.argtypes = [_i]
    L.wino_status_string.restype = ctypes.c_char_p
    for name in EXPORTED:
        getattr(L, name)  # every declared entry point must resolve
    _libs[path] = L
    if path == LIB_PATH:
        _lib = L
    return L


def _status_string(s: int) -> str:
    try:
        return load_library().wino_status_string(s).decode()
    except OSError:
        return "status"


def _stream_handle(stream: Optional[torch.cuda.Stream]) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _dtype_code(dt: torch.dtype) -> int:
    if dt == torch.bfloat16:
        return BF16
    if dt == torch.float32:
        return F32
    raise ValueError("unsupported dtype %s" % dt)


class Plan:
    """A wino_plan: transforms of F(m,3) for the given points and scales.

    Options (wino_opts): y_path / gemm select the Y route and the GEMM kernel (AUTO by default);
    debug enables the dumps; y_groups selects the Y grouping (TILE, the default reading, or TAP);
    x_int8 and int8_transforms select the alternative input-side readings (int8 x per pixel
    group before the transform; int8 B^T and A^T with one scale per matrix)."""

    def __init__(self, m: int, points: Sequence[float], S_B=None, S_G=None, group: int = 32,
                 y_path: int = YPATH_AUTO, gemm: int = GEMM_AUTO, debug: int = 0, y_groups: int = YGROUPS_TILE,
                 x_int8: bool = False, int8_transforms: bool = False, variant: str = "release",
                 fused: int = FUSED_AUTO):
        L = load_library(variant=variant)
        self._L = L
        n = m + 2
        pts = (ctypes.c_double * n)(*[float(p) for p in points])
        sb = None if S_B is None else (ctypes.c_float * n)(*[float(v) for v in S_B])
        sg = None if S_G is None else (ctypes.c_float * n)(*[float(v) for v in S_G])
        opts = Opts(y_path, gemm, debug, y_groups, int(x_int8), int(int8_transforms), int(fused))
        h = _vp()
        rc = L.wino_plan(ctypes.byref(h), m, pts, sb, sg, group, ctypes.byref(opts))
        if rc != OK:
            raise WinoError(rc, "wino_plan")
        self._h = h
        self.m, self.n, self.group, self.y_groups = m, n, group, y_groups

    def __del__(self):
        h = getattr(self, "_h", None)
        L = getattr(self, "_L", None)
        if h is not None and L is not None:
            L.wino_plan_destroy(h)
            self._h = None

    def _check(self, rc: int, what: str):
        if rc != OK:
            raise WinoError(rc, what, self._L.wino_last_cuda_error(self._h))

    # -------------------------------------------------------------- queries
    def matrices(self):
        n, m = self.n, self.m
        BT = (ctypes.c_float * (n * n))()
        G = (ctypes.c_double * (n * 3))()
        AT = (ctypes.c_float * (m * n))()
        self._check(self._L.wino_plan_matrices(self._h, BT, G, AT), "wino_plan_matrices")
        import numpy as np
        return (np.array(BT, dtype=np.float32).reshape(n, n), np.array(G, dtype=np.float64).reshape(n, 3),
                np.array(AT, dtype=np.float32).reshape(m, n))

    def weight_bytes(self, Cin: int, Cout: int) -> int:
        return int(self._L.wino_weight_bytes(self._h, Cin, Cout))

    def workspace_bytes(self, N: int, H: int, W: int, Cin: int, Cout: int) -> int:
        return int(self._L.wino_workspace_bytes(self._h, N, H, W, Cin, Cout))

    def host_staging_bytes(self, N, H, W, Cin, Cout, x_dtype=torch.bfloat16, y_dtype=torch.bfloat16) -> int:
        return int(self._L.wino_host_staging_bytes(self._h, N, H, W, Cin, Cout, _dtype_code(x_dtype),
                                                _dtype_code(y_dtype)))

    def resolved_config(self, N, H, W, Cin, Cout):
        yp, gm = _i(), _i()
        self._check(self._L.wino_resolved_config(self._h, N, H, W, Cin, Cout, ctypes.byref(yp), ctypes.byref(gm)),
                    "wino_resolved_config")
        return yp.value, gm.value

    def resolved_variants(self, N, H, W, Cin, Cout) -> int:
        """Bit set of VARIANT_* the call of this shape runs (same bytes in every variant)."""
        f = _i()
        self._check(self._L.wino_resolved_variants(self._h, N, H, W, Cin, Cout, ctypes.byref(f)),
                    "wino_resolved_variants")
        return f.value

    def launches_per_call(self, N, H, W, Cin, Cout) -> int:
        return int(self._L.wino_launches_per_call(self._h, N, H, W, Cin, Cout))

    # ---------------------------------------------------------------- calls
    def transform_weights(self, w: torch.Tensor, out: Optional[torch.Tensor] = None, stream=None) -> torch.Tensor:
        """w: fp32 [Cout][3][3][Cin] on the GPU -> uint8 buffer of wino_weight_bytes."""
        assert w.is_cuda and w.dtype == torch.float32 and w.is_contiguous() and w.dim() == 4
        Cout, _, _, Cin = w.shape
        nbytes = self.weight_bytes(Cin, Cout)
        if nbytes == 0:
            raise WinoError(ERR_INVALID_ARG, "wino_weight_bytes")
        if out is None:
            out = torch.empty(nbytes, dtype=torch.uint8, device=w.device)
        self._check(self._L.wino_transform_weights(self._h, w.data_ptr(), Cin, Cout, out.data_ptr(), out.numel(),
                                                _stream_handle(stream)), "wino_transform_weights")
        return out

    def conv2d(self, x: torch.Tensor, wt: torch.Tensor, Cout: int, out_dtype: torch.dtype = torch.bfloat16,
               out: Optional[torch.Tensor] = None, workspace: Optional[torch.Tensor] = None,
               stream=None) -> torch.Tensor:
        """x: [N][H][W][Cin] bf16/fp32 NHWC on the GPU; wt from transform_weights."""
        assert x.is_cuda and x.is_contiguous() and x.dim() == 4
        N, H, W, Cin = x.shape
        if out is None:
            out = torch.empty((N, H, W, Cout), dtype=out_dtype, device=x.device)
        need = self.workspace_bytes(N, H, W, Cin, Cout)
        if need == 0:
            raise WinoError(ERR_INVALID_ARG, "wino_workspace_bytes")
        if workspace is None:
            workspace = torch.empty(need, dtype=torch.uint8, device=x.device)
        self._check(self._L.wino_conv2d_int8(self._h, x.data_ptr(), _dtype_code(x.dtype), N, H, W, Cin, wt.data_ptr(),
                                          Cout, out.data_ptr(), _dtype_code(out.dtype), workspace.data_ptr(),
                                          workspace.numel(), _stream_handle(stream)), "wino_conv2d_int8")
        return out

    def conv2d_noalloc(self, x: torch.Tensor, wt: torch.Tensor, Cout: int, out: torch.Tensor, stream=None):
        """wino_conv2d_int8_noalloc: no workspace argument; the library's fixed
        device scratch array is used instead (see include/wino.h)."""
        N, H, W, Cin = x.shape
        self._check(self._L.wino_conv2d_int8_noalloc(self._h, x.data_ptr(), _dtype_code(x.dtype), N, H, W, Cin,
                                                  wt.data_ptr(), Cout, out.data_ptr(), _dtype_code(out.dtype),
                                                  _stream_handle(stream)), "wino_conv2d_int8_noalloc")
        return out

    def conv2d_host(self, x_host: torch.Tensor, wt: torch.Tensor, Cout: int, y_host: torch.Tensor,
                    workspace: torch.Tensor, stream=None):
        """Host (pinned) input and output; copies happen inside the call, asynchronously."""
        N, H, W, Cin = x_host.shape
        self._check(self._L.wino_conv2d_int8_host(self._h, x_host.data_ptr(), _dtype_code(x_host.dtype), N, H, W, Cin,
                                               wt.data_ptr(), Cout, y_host.data_ptr(), _dtype_code(y_host.dtype),
                                               workspace.data_ptr(), workspace.numel(), _stream_handle(stream)),
                    "wino_conv2d_int8_host")

    def profile_begin(self, max_calls: int):
        """Record per-kernel CUDA events on the launching stream for the next max_calls calls."""
        self._check(self._L.wino_profile_begin(self._h, max_calls), "wino_profile_begin")

    def profile_end(self):
        """-> (summed ms per launch index, calls recorded)."""
        ms = (ctypes.c_float * 8)()
        nl, nc = _i(), _i()
        self._check(self._L.wino_profile_end(self._h, ms, 8, ctypes.byref(nl), ctypes.byref(nc)), "wino_profile_end")
        return [ms[i] for i in range(min(nl.value, 8))], nc.value

    def check_device_error(self, workspace: torch.Tensor, N, H, W, Cin, Cout, stream=None) -> int:
        return self._L.wino_check_device_error(self._h, workspace.data_ptr(), N, H, W, Cin, Cout, _stream_handle(stream))

    def check_guards(self, workspace: torch.Tensor, N, H, W, Cin, Cout, stream=None):
        """(status, index of the first overwritten guard band or -1) after the last conv2d call."""
        bad = _i()
        rc = self._L.wino_check_guards(self._h, workspace.data_ptr(), N, H, W, Cin, Cout, _stream_handle(stream),
                                       ctypes.byref(bad))
        return rc, bad.value

    def check_device_error_noalloc(self, N, H, W, Cin, Cout, stream=None) -> int:
        """The device error word of the last conv2d_noalloc call of this shape (in the library's scratch)."""
        return self._L.wino_check_device_error_noalloc(self._h, N, H, W, Cin, Cout, _stream_handle(stream))

    def debug_dump(self, workspace: torch.Tensor, N, H, W, Cin, Cout, what: int):
        """Copy one intermediate tensor of the last call (logical layout, see include/wino.h)."""
        import numpy as np
        m, n2, G = self.m, self.n * self.n, self.group
        T = N * math.ceil(H / m) * math.ceil(W / m)
        shapes = {DUMP_VQ: ((T, n2, Cin), np.int8), DUMP_SV: ((T, n2, Cin // G), np.float32),
                  DUMP_YQ: ((T, n2, Cout), np.int8),
                  DUMP_SY: (((T, n2, Cout // G) if self.y_groups == YGROUPS_TAP else (T, Cout // G)), np.float32),
                  DUMP_Y32: ((T, n2, Cout), np.float32), DUMP_ACC32: ((n2, T, Cout, Cin // G), np.int32)}
        shape, dt = shapes[what]
        a = np.zeros(shape, dt)
        self._check(self._L.wino_debug_dump(self._h, workspace.data_ptr(), N, H, W, Cin, Cout, what,
                                         a.ctypes.data, a.nbytes), "wino_debug_dump")
        return a
