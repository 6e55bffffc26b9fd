"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every entry point include/wino.h declares, and its host plan (transform
construction, argument checks, workspace sizing) behaves as specified."""
import ctypes
import math
import os
import re

import numpy as np
import pytest

import oracle
from group_wise_int8_b200 import build, synth, wino

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return wino.load_library()


def declared_functions():
    src = open(os.path.join(ROOT, "include", "wino.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(wino_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_entry_points():
    assert declared_functions() == sorted(wino.EXPORTED)


def test_binding_constants_match_the_header():
    src = open(os.path.join(ROOT, "include", "wino.h")).read()
    m = re.search(r"#define WINO_NOALLOC_SCRATCH_BYTES \((\d+)u << (\d+)\)", src)
    assert m and int(m.group(1)) << int(m.group(2)) == wino.NOALLOC_SCRATCH_BYTES


def test_noalloc_error_query_checks_its_arguments(lib):
    """wino_check_device_error_noalloc rejects a null plan, bad shapes and shapes beyond the
    scratch array before touching the GPU."""
    assert lib.wino_check_device_error_noalloc(None, 1, 8, 8, 32, 32, None) == wino.ERR_INVALID_ARG
    plan = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    assert lib.wino_check_device_error_noalloc(plan._h, 1, 8, 8, 33, 32, None) == wino.ERR_INVALID_ARG
    assert lib.wino_check_device_error_noalloc(plan._h, 128, 56, 56, 64, 64, None) == wino.ERR_WORKSPACE


@pytest.mark.parametrize("variant", ["release", "debug"])
def test_library_exports_every_declared_symbol(lib, variant):
    L = wino.load_library(variant=variant)
    for name in declared_functions():
        assert hasattr(L, name), name
    out = os.popen("nm -D --defined-only %s" % wino.LIB_PATHS[variant]).read()
    for name in declared_functions():
        assert re.search(r"\bT %s\b" % name, out), name


@pytest.mark.parametrize("m,pts", [(4, synth.POINTS_F4), (6, synth.POINTS_F6)])
@pytest.mark.parametrize("scales", ["identity", "loguniform", "rownorm"])
def test_plan_matches_oracle_bit_exactly(lib, m, pts, scales):
    """The library builds V^{-1} from Lagrange basis polynomials, the oracle by
    Gauss-Jordan elimination; both round the same exact rationals once."""
    n = m + 2
    sb = sg = None
    if scales == "loguniform":
        r = np.random.default_rng(m)
        sb = np.exp(r.uniform(math.log(0.5), math.log(2), n)).astype(np.float32)
        sg = np.exp(r.uniform(math.log(0.5), math.log(2), n)).astype(np.float32)
    elif scales == "rownorm":
        p0 = oracle.Plan(m, pts)
        sb = (1.0 / np.linalg.norm(p0.BT_d, axis=1)).astype(np.float32)
        sg = (1.0 / np.linalg.norm(p0.G_d, axis=1)).astype(np.float32)
    op = oracle.Plan(m, pts, sb, sg)
    BT, G, AT = wino.Plan(m, pts, sb, sg, 32).matrices()
    assert np.array_equal(BT.view(np.uint32), op.BT_f.view(np.uint32))
    assert np.array_equal(G.view(np.uint64), op.G_d.view(np.uint64))
    assert np.array_equal(AT.view(np.uint32), op.AT_f.view(np.uint32))


def test_plan_other_point_orders_match_oracle(lib):
    pts = (math.inf, 0.5, -2.0, 1.0, 0.0, -1.0)   # permuted F(4,3) points: generic (unmasked) kernels
    op = oracle.Plan(4, pts)
    BT, G, AT = wino.Plan(4, pts, None, None, 64).matrices()
    assert np.array_equal(BT, op.BT_f) and np.array_equal(G, op.G_d) and np.array_equal(AT, op.AT_f)


@pytest.mark.parametrize("pts", [synth.POINTS_F2, (math.inf, -1.0, 0.0, 1.0)])
def test_plan_f23_matches_oracle(lib, pts):
    op = oracle.Plan(2, pts)
    BT, G, AT = wino.Plan(2, pts, None, None, 32).matrices()
    assert np.array_equal(BT, op.BT_f) and np.array_equal(G, op.G_d) and np.array_equal(AT, op.AT_f)


@pytest.mark.parametrize("m,pts,scaled", [(2, synth.POINTS_F2, False), (4, synth.POINTS_F4, True),
                                          (6, synth.POINTS_F6, False), (6, synth.POINTS_F6, True)])
def test_plan_int8_transforms_match_oracle(lib, m, pts, scaled):
    """The int8-transform reading is applied at plan time on the host: the library's B^T
    and A^T equal the oracle's quantised matrices bit for bit, G is untouched."""
    n = m + 2
    r = np.random.default_rng(m)
    sb = (r.integers(32, 129, n) / 64.0).astype(np.float32) if scaled else None
    sg = (r.integers(32, 129, n) / 64.0).astype(np.float32) if scaled else None
    op = oracle.Plan(m, pts, sb, sg, int8_transforms=True)
    BT, G, AT = wino.Plan(m, pts, sb, sg, 32, int8_transforms=True).matrices()
    assert np.array_equal(BT, op.BT_f) and np.array_equal(G, op.G_d) and np.array_equal(AT, op.AT_f)
    BT0, _, AT0 = wino.Plan(m, pts, sb, sg, 32).matrices()
    assert not np.array_equal(BT0, BT)


def test_short_layers_take_the_fp32_y_path(lib):
    """At most 80 tiles with Cout a multiple of 128: AUTO resolves to the fp32-Y path (whose GEMM
    pass runs with swapped operands); an explicit recompute request is kept."""
    auto = wino.Plan(6, synth.POINTS_F6, None, None, 64)
    assert auto.resolved_config(2, 8, 8, 1280, 1280)[0] == wino.YPATH_Y32          # T = 8
    assert auto.resolved_config(2, 16, 16, 1280, 1280)[0] == wino.YPATH_Y32        # T = 18
    for n, swapped in ((8, True), (9, False)):                                       # T = 72, 81
        assert bool(auto.resolved_variants(n, 16, 16, 1280, 1280) & wino.VARIANT_SWAPPED_GEMM) == swapped
    assert auto.resolved_variants(8, 16, 16, 1280, 320) & wino.VARIANT_SWAPPED_GEMM == 0   # Cout % 128 != 0
    rec = wino.Plan(6, synth.POINTS_F6, None, None, 64, y_path=wino.YPATH_RECOMPUTE)
    assert rec.resolved_config(2, 8, 8, 1280, 1280)[0] == wino.YPATH_RECOMPUTE
    assert rec.launches_per_call(2, 8, 8, 1280, 1280) == 4
    assert auto.launches_per_call(2, 8, 8, 1280, 1280) == 3


def test_x_int8_option_adds_a_launch_and_workspace(lib):
    shape = (2, 20, 20, 64, 64)
    p0 = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    p1 = wino.Plan(6, synth.POINTS_F6, None, None, 32, x_int8=True)
    assert p1.launches_per_call(*shape) == p0.launches_per_call(*shape) + 1
    assert p1.workspace_bytes(*shape) >= p0.workspace_bytes(*shape) + 4 * 2 * 20 * 20 * 64
    for bad in (dict(x_int8=2), dict(int8_transforms=-1)):
        with pytest.raises(wino.WinoError) as e:
            wino.Plan(6, synth.POINTS_F6, None, None, 32, **bad)
        assert e.value.status == wino.ERR_INVALID_ARG


@pytest.mark.parametrize("bad", [
    dict(m=5), dict(group=48), dict(points=(0.0, 1.0, 1.0, 2.0, -2.0, math.inf)),
    dict(points=(0.0, 1.0, -1.0, math.inf, -2.0, math.inf)), dict(points=(0.0, 1.0, -1.0, 2.0, float("nan"), math.inf)),
    dict(S_B=[1, 1, 0, 1, 1, 1]),
])
def test_plan_rejects_invalid_arguments(lib, bad):
    kw = dict(m=4, points=synth.POINTS_F4, S_B=None, S_G=None, group=32)
    kw.update(bad)
    if kw["m"] != 4:
        kw["points"] = kw["points"] + (0.5,) * (kw["m"] - 4)
    with pytest.raises(wino.WinoError) as e:
        wino.Plan(kw["m"], kw["points"], kw["S_B"], kw["S_G"], kw["group"])
    assert e.value.status == wino.ERR_INVALID_ARG


def test_y_groups_option(lib):
    tap = wino.Plan(6, synth.POINTS_F6, None, None, 32, y_groups=wino.YGROUPS_TAP)
    assert tap.resolved_config(32, 56, 56, 64, 64)[0] == wino.YPATH_Y32     # the per-tap reading needs fp32 Y
    for bad in (dict(y_groups=2), dict(y_groups=wino.YGROUPS_TAP, y_path=wino.YPATH_RECOMPUTE)):
        with pytest.raises(wino.WinoError) as e:
            wino.Plan(6, synth.POINTS_F6, None, None, 32, **bad)
        assert e.value.status == wino.ERR_INVALID_ARG


def test_workspace_and_weight_sizes(lib):
    p = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    N, H, W, C = 32, 56, 56, 64
    T = N * 10 * 10
    ws = p.workspace_bytes(N, H, W, C, C)
    Tpad = (T + 127) // 128 * 128
    assert ws >= Tpad * 64 * C + 4 * 64 * (C // 32) * Tpad + 4 * Tpad * (C // 32) + T * 64 * C
    assert p.weight_bytes(C, C) >= 64 * C * C + 4 * 64 * (C // 32) * C
    assert p.workspace_bytes(N, H, W, 48, C) == 0       # Cin not a multiple of G
    assert p.weight_bytes(C, 40) == 0


def test_resolved_config_auto_is_fp32_y(lib):
    """AUTO resolves to the single-pass fp32-Y path on every shape (measured faster than the
    two-pass recompute path on each configured layer); recompute runs on request."""
    p = wino.Plan(6, synth.POINTS_F6, None, None, 64)
    for shape in ((32, 56, 56, 64, 64), (64, 28, 28, 128, 128), (2, 64, 64, 320, 320), (8, 32, 32, 1920, 640),
                  (2, 8, 8, 1280, 1280)):
        assert p.resolved_config(*shape)[0] == wino.YPATH_Y32, shape
        assert p.launches_per_call(*shape) == 3
    rec = wino.Plan(6, synth.POINTS_F6, None, None, 64, y_path=wino.YPATH_RECOMPUTE)
    assert rec.resolved_config(32, 56, 56, 64, 64)[0] == wino.YPATH_RECOMPUTE
    assert rec.launches_per_call(32, 56, 56, 64, 64) == 4
    assert p.resolved_config(2, 8, 8, 1280, 1280)[1] == wino.GEMM_TCGEN05
    forced = wino.Plan(6, synth.POINTS_F6, None, None, 64, y_path=wino.YPATH_RECOMPUTE, gemm=wino.GEMM_SIMT)
    assert forced.resolved_config(2, 8, 8, 1280, 1280) == (wino.YPATH_RECOMPUTE, wino.GEMM_SIMT)
    assert forced.launches_per_call(2, 8, 8, 1280, 1280) == 4


def test_parity_cases_cover_every_kernel_variant(lib):
    """The GPU parity cases (stagewise, both Y paths) run each shape-chosen variant -- swapped GEMM,
    split input and split output transforms, the A-resident GEMM walk -- and also each kernel it
    replaces, so bit-exactness is checked on both sides of every choice (SM count 148, as on the
    B200)."""
    from tests.test_gpu_parity import CASES
    seen = {}
    for name, (m, pts, N, H, W, Cin, Cout, G, *_rest) in CASES.items():
        for y_path in (wino.YPATH_RECOMPUTE, wino.YPATH_Y32):
            flags = wino.Plan(m, pts, None, None, G, y_path=y_path).resolved_variants(N, H, W, Cin, Cout)
            for bit in (wino.VARIANT_SWAPPED_GEMM, wino.VARIANT_SPLIT_INPUT, wino.VARIANT_SPLIT_OUTPUT,
                        wino.VARIANT_A_RESIDENT):
                seen.setdefault(bit, set()).add(bool(flags & bit))
    assert all(v == {False, True} for v in seen.values()), seen


def test_variants_follow_the_shape(lib):
    p = wino.Plan(6, synth.POINTS_F6, None, None, 64)
    # SD-shaped C1280 8x8, N2: 8 tiles -> all three variants
    assert p.resolved_variants(2, 8, 8, 1280, 1280) == (wino.VARIANT_SWAPPED_GEMM | wino.VARIANT_SPLIT_INPUT |
                                                        wino.VARIANT_SPLIT_OUTPUT)
    q = wino.Plan(6, synth.POINTS_F6, None, None, 32)
    assert q.resolved_variants(32, 56, 56, 64, 64) == 0          # the default layer: none
    # SD-shaped 64x64 and 32x32 layers: several column blocks, A resident up to Cin 960 (four K stages
    # beside three B stages); Cin 1920 does not fit
    for plan, shape, ar in ((p, (8, 64, 64, 320, 320), True), (p, (8, 64, 64, 960, 320), True),
                            (p, (8, 32, 32, 640, 640), True), (p, (8, 32, 32, 1920, 640), False)):
        assert bool(plan.resolved_variants(*shape) & wino.VARIANT_A_RESIDENT) == ar, shape
