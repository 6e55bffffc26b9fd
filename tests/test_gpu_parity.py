"""GPU parity: the CUDA path through the C ABI against the CPU oracle on the
same seeded inputs.

Bar (from the method's specification of this library): every int8 tensor
(Uq, Vq, Yq), every scale (sU, sV, sY), the int32 per-K-group accumulators and
the fp32 Y are bit-exact; fp32 outputs agree within 1e-5 relative L2; the
SQNR against the fp64 direct convolution equals the oracle's to 0.01 dB.  The
kernels evaluate every fp32 chain in the oracle's order, so the outputs are in
fact compared element by element (equal values), with the norm and the SQNR
kept as secondary checks.
Zero-coefficient skipping in the transforms can change only the sign of a
zero, which the quantiser maps to the same code, so value equality is the
bit-exactness criterion for the fp32 tensors.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth, wino
from tests.gpu_util import assert_bits_equal, bf16_round, rel_l2, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

P2, P4, P6 = synth.POINTS_F2, synth.POINTS_F4, synth.POINTS_F6

# name: (m, points, N, H, W, Cin, Cout, G, dtype, act, scales)
CASES = {
    "tiny_f4": (4, P4, 1, 16, 16, 32, 32, 32, "f32", "normal", "identity"),
    "ragged_f6_cout96": (6, P6, 2, 13, 11, 64, 96, 32, "bf16", "relu_normal", "loguniform"),
    "f4_g64_outliers": (4, P4, 1, 20, 20, 128, 64, 64, "bf16", "student_t_outliers", "loguniform"),
    "f6_g64_cout128": (6, P6, 1, 12, 12, 64, 128, 64, "bf16", "student_t_outliers", "loguniform"),
    "f6_g256": (6, P6, 1, 8, 8, 256, 256, 256, "bf16", "relu_normal", "loguniform"),
    "f6_wide_k": (6, P6, 1, 8, 8, 1280, 128, 64, "bf16", "student_t_outliers", "loguniform"),
    "f4_two_row_blocks": (4, P4, 2, 40, 38, 64, 64, 32, "bf16", "relu_normal", "loguniform"),
    "f6_single_partial_tile": (6, P6, 1, 3, 5, 32, 32, 32, "f32", "normal", "loguniform"),
    "f6_one_pixel": (6, P6, 3, 1, 1, 64, 32, 32, "bf16", "relu_normal", "identity"),
    "f4_permuted_points": (4, (math.inf, 0.5, -2.0, 1.0, 0.0, -1.0), 1, 10, 9, 64, 64, 64, "bf16",
                           "relu_normal", "loguniform"),
    "f2_ragged": (2, P2, 2, 13, 11, 64, 64, 32, "bf16", "relu_normal", "loguniform"),
    "f2_g64_cout128_f32": (2, P2, 1, 30, 30, 128, 128, 64, "f32", "student_t_outliers", "loguniform"),
    "f2_permuted_points": (2, (math.inf, -1.0, 0.0, 1.0), 1, 9, 10, 32, 64, 32, "bf16", "normal", "loguniform"),
    # enough (tile, channel pair) items for the one-thread-per-item fp32-Y output kernel; the
    # smaller cases take the split kernel on that path
    "f6_many_items": (6, P6, 4, 60, 59, 64, 256, 64, "bf16", "relu_normal", "loguniform"),
    # enough tiles per channel group for the one-thread-per-item input transform (the smaller
    # cases take its split kernel)
    "f6_many_tiles": (6, P6, 24, 56, 56, 64, 32, 32, "bf16", "relu_normal", "loguniform"),
    # the widest concatenated-skip conv of the SD-shaped stack: 40 K-groups per tap
    "f6_cin2560_cout1280": (6, P6, 2, 16, 16, 2560, 1280, 64, "bf16", "student_t_outliers", "loguniform"),
    # the swapped fp32-Y pass at each of its wider MMA N: 45 tiles (N 48), 64 tiles (N 64), 72 tiles
    # of ragged images with a ragged last K stage (N 80), exactly 80 tiles, and 81 tiles (not swapped)
    "f6_swap_n48": (6, P6, 5, 16, 16, 256, 256, 64, "bf16", "relu_normal", "loguniform"),
    "f4_swap_n64": (4, P4, 1, 30, 30, 128, 128, 32, "f32", "normal", "loguniform"),
    "f6_swap_n80_ragged": (6, P6, 2, 34, 35, 320, 256, 64, "bf16", "student_t_outliers", "loguniform"),
    "f4_swap_n80_full": (4, P4, 5, 16, 16, 128, 128, 64, "bf16", "relu_normal", "loguniform"),
    "f6_81_tiles": (6, P6, 1, 54, 54, 128, 128, 64, "bf16", "relu_normal", "loguniform"),
    # the A-resident GEMM walk: a tap's A tile kept across three column blocks, over two K stages (the
    # second ragged: 5 groups as 4 + 1), and over four K stages across two column blocks
    "f6_a_resident_ragged_k": (6, P6, 2, 40, 40, 320, 192, 64, "bf16", "student_t_outliers", "loguniform"),
    "f6_a_resident_cin960": (6, P6, 1, 60, 60, 960, 128, 64, "bf16", "relu_normal", "loguniform"),
}


def make_case(name, seed=0):
    m, pts, N, H, W, Cin, Cout, G, dtype, act, scales = CASES[name]
    layer = synth.random_layer(seed, m, N, H, W, Cin, Cout, G, dtype=dtype, act=act, scales=scales,
                               w_var_num=2.0, workload="parity_" + name)
    x_f32, x_bits = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    return m, pts, G, x_f32, x_bits, w, sb, sg


_oracle_cache = {}


def oracle_for(name):
    if name not in _oracle_cache:
        m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
        _oracle_cache[name] = run_oracle(m, pts, sb, sg, G, x_f32, w, want_acc=True)
    return _oracle_cache[name]


@pytest.mark.parametrize("gemm", [wino.GEMM_TCGEN05, wino.GEMM_SIMT])
@pytest.mark.parametrize("y_path", [wino.YPATH_RECOMPUTE, wino.YPATH_Y32])
@pytest.mark.parametrize("name", list(CASES))
def test_stagewise_bit_exact(cuda_dev, name, y_path, gemm):
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
    ref = oracle_for(name)
    got = run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=torch.float32, y_path=y_path, gemm=gemm,
                  debug=wino.DEBUG_YQ | wino.DEBUG_ACC32)
    assert got["gemm"] == gemm and got["y_path"] == y_path
    for k in ("Uq", "sU", "Vq", "sV", "acc", "Yq", "sY"):
        assert_bits_equal(k, got[k], ref[k])
    if y_path == wino.YPATH_Y32:
        assert_bits_equal("Y", got["Y"], ref["Y"])
    assert_bits_equal("out", got["out"], ref["out"])
    assert rel_l2(got["out"], ref["out"]) <= 1e-5
    s_gpu, s_orc = oracle.sqnr_db(ref["ref"], got["out"]), oracle.sqnr_db(ref["ref"], ref["out"])
    assert abs(s_gpu - s_orc) <= 0.01


_oracle_tap_cache = {}


@pytest.mark.parametrize("gemm", [wino.GEMM_TCGEN05, wino.GEMM_SIMT])
@pytest.mark.parametrize("name", ["ragged_f6_cout96", "f4_g64_outliers", "f6_g256", "f6_single_partial_tile",
                                  "f2_ragged", "f4_permuted_points"])
def test_y_tap_reading_bit_exact(cuda_dev, name, gemm):
    """The per-tap Y groups (WINO_YGROUPS_TAP): Yq and the [T][n2][Cout/G] scales bit for bit,
    the output within the fp32 tolerance, on the fp32-Y path it forces."""
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
    if name not in _oracle_tap_cache:
        _oracle_tap_cache[name] = run_oracle(m, pts, sb, sg, G, x_f32, w, per_tap=True)
    ref = _oracle_tap_cache[name]
    got = run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=torch.float32, gemm=gemm,
                  debug=wino.DEBUG_YQ, y_groups=wino.YGROUPS_TAP)
    assert got["y_path"] == wino.YPATH_Y32
    for k in ("Vq", "sV", "Y", "Yq", "sY"):
        assert_bits_equal(k, got[k], ref[k])
    assert_bits_equal("out", got["out"], ref["out"])
    assert rel_l2(got["out"], ref["out"]) <= 1e-5
    assert abs(oracle.sqnr_db(ref["ref"], got["out"]) - oracle.sqnr_db(ref["ref"], ref["out"])) <= 0.01


_oracle_alt_cache = {}
_ALT = {"x_int8": dict(x_int8=True), "int8_transforms": dict(int8_transforms=True),
        "both": dict(x_int8=True, int8_transforms=True)}


@pytest.mark.parametrize("y_path", [wino.YPATH_RECOMPUTE, wino.YPATH_Y32])
@pytest.mark.parametrize("reading", list(_ALT))
@pytest.mark.parametrize("name", ["tiny_f4", "ragged_f6_cout96", "f4_g64_outliers", "f6_g256", "f2_ragged",
                                  "f6_one_pixel"])
def test_alternative_input_readings_bit_exact(cuda_dev, name, reading, y_path):
    """x group-quantised per pixel before the transform (x_int8) and/or int8 B^T and A^T with
    one scale per matrix (int8_transforms): every code and scale bit for bit, the output
    within the fp32 tolerance, on both Y paths."""
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
    key = (name, reading)
    if key not in _oracle_alt_cache:
        _oracle_alt_cache[key] = run_oracle(m, pts, sb, sg, G, x_f32, w, **_ALT[reading])
    ref = _oracle_alt_cache[key]
    got = run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=torch.float32, y_path=y_path,
                  debug=wino.DEBUG_YQ, **_ALT[reading])
    keys = ("Uq", "sU", "Vq", "sV", "Yq", "sY") + (("Y",) if y_path == wino.YPATH_Y32 else ())
    for k in keys:
        assert_bits_equal(k, got[k], ref[k])
    assert_bits_equal("out", got["out"], ref["out"])
    assert rel_l2(got["out"], ref["out"]) <= 1e-5
    assert abs(oracle.sqnr_db(ref["ref"], got["out"]) - oracle.sqnr_db(ref["ref"], ref["out"])) <= 0.01


def test_y_tap_rejects_recompute_path(cuda_dev):
    with pytest.raises(wino.WinoError):
        wino.Plan(6, P6, None, None, 32, y_path=wino.YPATH_RECOMPUTE, y_groups=wino.YGROUPS_TAP)


@pytest.mark.parametrize("name", ["ragged_f6_cout96", "f6_g64_cout128", "f4_two_row_blocks"])
def test_default_path_bf16_output(cuda_dev, name):
    """Default options (AUTO path and kernel) with bf16 output, as the benchmark runs them."""
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case(name)
    ref = oracle_for(name)
    got = run_gpu(m, pts, sb, sg, G, x_f32, x_bits, w, out_dtype=torch.bfloat16)
    assert got["gemm"] == wino.GEMM_TCGEN05
    want = bf16_round(ref["out"])
    assert_bits_equal("out", got["out"], want)
    assert abs(oracle.sqnr_db(ref["ref"], got["out"]) - oracle.sqnr_db(ref["ref"], want)) <= 0.01


def test_host_entry_point_matches_device_call(cuda_dev):
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case("ragged_f6_cout96")
    N, H, W, Cin = x_f32.shape
    Cout = w.shape[0]
    plan = wino.Plan(m, pts, sb, sg, G)
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    x_host = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((N, H, W, Cout), dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) + plan.host_staging_bytes(N, H, W, Cin, Cout),
                     dtype=torch.uint8, device="cuda")
    plan.conv2d_host(x_host, wt, Cout, y_host, ws)
    torch.cuda.synchronize()
    y_dev = plan.conv2d(x_host.cuda(), wt, Cout, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())


@pytest.mark.parametrize("x_int8", [False, True])
@pytest.mark.parametrize("N", [3, 5, 9])
def test_host_entry_point_chunks_match_device_call(cuda_dev, N, x_int8):
    """The host entry point pipelines chunks of images; its bytes equal one device call (also
    with the int8-x reading, whose fp32 copy of x lives in each chunk's workspace)."""
    layer = synth.random_layer(4, 6, N, 14, 13, 64, 64, 32, dtype="f32", act="relu_normal",
                               scales="loguniform", workload="host_chunks")
    x_f32, _ = synth.make_input(layer)
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    plan = wino.Plan(6, P6, sb, sg, 32, x_int8=x_int8)
    H, W, Cin, Cout = 14, 13, 64, 64
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    x_host = torch.from_numpy(x_f32).pin_memory()
    y_host = torch.empty((N, H, W, Cout), dtype=torch.float32).pin_memory()
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) +
                     plan.host_staging_bytes(N, H, W, Cin, Cout, torch.float32, torch.float32),
                     dtype=torch.uint8, device="cuda")
    ws.fill_(0x5A)
    plan.conv2d_host(x_host, wt, Cout, y_host, ws)
    torch.cuda.synchronize()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    y_dev = plan.conv2d(x_host.cuda(), wt, Cout, out_dtype=torch.float32)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_host_entry_point_last_chunk_on_another_kernel(cuda_dev):
    """N = 8 in chunks of 3, 3 and 2 images: on this SD-shaped layer (320 -> 640, 32x32, G = 64)
    the 3-image chunks (108 tiles) run the GEMM with tiles on the MMA rows and the 2-image chunk
    (72 tiles) the swapped GEMM; the chunk workspaces are carved for every chunk size."""
    N, H, W, Cin, Cout = 8, 32, 32, 320, 640
    layer = synth.random_layer(11, 6, N, H, W, Cin, Cout, 64, dtype="bf16", act="student_t_outliers",
                               w_var_num=1.0, workload="host_chunk_paths")
    sb, sg = synth.make_scales(layer)
    plan = wino.Plan(6, P6, sb, sg, 64)
    assert not plan.resolved_variants(3, H, W, Cin, Cout) & wino.VARIANT_SWAPPED_GEMM
    assert plan.resolved_variants(2, H, W, Cin, Cout) & wino.VARIANT_SWAPPED_GEMM
    wt = plan.transform_weights(torch.from_numpy(synth.make_weights(layer)).cuda())
    _, bits = synth.make_input(layer)
    x_host = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory()
    y_host = torch.empty((N, H, W, Cout), dtype=torch.bfloat16).pin_memory()
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) + plan.host_staging_bytes(N, H, W, Cin, Cout),
                     dtype=torch.uint8, device="cuda")
    plan.conv2d_host(x_host, wt, Cout, y_host, ws)
    torch.cuda.synchronize()
    assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
    y_dev = plan.conv2d(x_host.cuda(), wt, Cout, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    assert torch.equal(y_host, y_dev.cpu())


def test_back_to_back_host_calls_overlap_safely(cuda_dev):
    """Consecutive host calls of one shape overlap (the next batch's input copies start before
    the previous call ends); with different inputs and outputs every call still gives the bytes
    of its own device call."""
    N, H, W, Cin, Cout = 8, 14, 13, 64, 64
    plan = wino.Plan(6, P6, None, None, 32)
    w = synth.make_weights(synth.random_layer(7, 6, N, H, W, Cin, Cout, 32, workload="host_b2b"))
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) +
                     plan.host_staging_bytes(N, H, W, Cin, Cout, torch.bfloat16, torch.bfloat16),
                     dtype=torch.uint8, device="cuda")
    xs, ys = [], []
    for seed in range(4):
        layer = synth.random_layer(100 + seed, 6, N, H, W, Cin, Cout, 32, dtype="bf16", act="relu_normal",
                                   workload="host_b2b")
        _, bits = synth.make_input(layer)
        xs.append(torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory())
        ys.append(torch.empty((N, H, W, Cout), dtype=torch.bfloat16).pin_memory())
    for _ in range(3):   # several rounds: later calls are chained to earlier ones
        for x_h, y_h in zip(xs, ys):
            plan.conv2d_host(x_h, wt, Cout, y_h, ws)
        torch.cuda.synchronize()
        assert plan.check_device_error(ws, N, H, W, Cin, Cout) == wino.OK
        for x_h, y_h in zip(xs, ys):
            y_dev = plan.conv2d(x_h.cuda(), wt, Cout, out_dtype=torch.bfloat16)
            torch.cuda.synchronize()
            assert torch.equal(y_h, y_dev.cpu())


def test_host_calls_of_two_plans_sharing_a_workspace(cuda_dev):
    """Two plans (layers of one shape) alternate host calls on one workspace: a call must not
    chain to its own plan's previous call across the other plan's call in between, whose
    convolution still reads the same staging buffers."""
    N, H, W, Cin, Cout = 6, 14, 13, 64, 64
    plans, wts, xs, ys = [], [], [], []
    ws = None
    for k in range(2):
        layer = synth.random_layer(200 + k, 6, N, H, W, Cin, Cout, 32, dtype="bf16", act="relu_normal",
                                   workload="host_two_plans")
        sb, sg = synth.make_scales(layer)
        plan = wino.Plan(6, P6, sb, sg, 32)
        plans.append(plan)
        wts.append(plan.transform_weights(torch.from_numpy(synth.make_weights(layer)).cuda()))
        _, bits = synth.make_input(layer)
        xs.append(torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).pin_memory())
        ys.append(torch.empty((N, H, W, Cout), dtype=torch.bfloat16).pin_memory())
        if ws is None:
            ws = torch.empty(plan.workspace_bytes(N, H, W, Cin, Cout) +
                             plan.host_staging_bytes(N, H, W, Cin, Cout, torch.bfloat16, torch.bfloat16),
                             dtype=torch.uint8, device="cuda")
    want = [plans[k].conv2d(xs[k].cuda(), wts[k], Cout, out_dtype=torch.bfloat16).cpu() for k in range(2)]
    for _ in range(4):
        for k in range(2):
            plans[k].conv2d_host(xs[k], wts[k], Cout, ys[k], ws)
    torch.cuda.synchronize()
    for k in range(2):
        assert torch.equal(ys[k], want[k]), k


@pytest.mark.parametrize("room", ["overlap", "tight"])
def test_host_calls_of_several_shapes_on_one_workspace(cuda_dev, room):
    """Back-to-back host calls cycling through three layers of different shapes and plans on one
    workspace, each call with its own input and output buffers and no synchronisation between
    calls: with room for two stagings above the largest convolution workspace every call's input
    copies overlap the previous call; on a workspace sized for the largest single call some calls
    find no clear staging and wait.  Every output equals the device entry point's."""
    shapes = [(6, 14, 13, 64, 64, 32), (4, 20, 20, 128, 64, 64), (3, 9, 10, 64, 128, 32)]
    plans, wts, need, stage = [], [], [], []
    for k, (N, H, W, Cin, Cout, G) in enumerate(shapes):
        layer = synth.random_layer(300 + k, 6, N, H, W, Cin, Cout, G, dtype="bf16", act="relu_normal",
                                   workload="host_shapes")
        sb, sg = synth.make_scales(layer)
        plan = wino.Plan(6, P6, sb, sg, G)
        plans.append(plan)
        wts.append(plan.transform_weights(torch.from_numpy(synth.make_weights(layer)).cuda()))
        need.append(plan.workspace_bytes(N, H, W, Cin, Cout))
        stage.append(plan.host_staging_bytes(N, H, W, Cin, Cout, torch.bfloat16, torch.bfloat16))
    size = max(need) + max(stage) if room == "overlap" else max(n + st for n, st in zip(need, stage))
    ws = torch.empty(size, dtype=torch.uint8, device="cuda")
    calls = []
    for rep in range(3):
        for k, (N, H, W, Cin, Cout, G) in enumerate(shapes):
            g = torch.Generator().manual_seed(1000 * rep + k)
            x = (torch.randn((N, H, W, Cin), generator=g) * (1 + rep)).to(torch.bfloat16).pin_memory()
            y = torch.full((N, H, W, Cout), float("nan"), dtype=torch.bfloat16).pin_memory()
            calls.append((k, x, y))
    for k, x, y in calls:
        plans[k].conv2d_host(x, wts[k], shapes[k][4], y, ws)
    torch.cuda.synchronize()
    k_last = calls[-1][0]   # the error word belongs to the last call's layout
    assert plans[k_last].check_device_error(ws, *shapes[k_last][:5]) == wino.OK
    for i, (k, x, y) in enumerate(calls):
        want = plans[k].conv2d(x.cuda(), wts[k], shapes[k][4], out_dtype=torch.bfloat16).cpu()
        assert torch.equal(y.view(torch.int16), want.view(torch.int16)), i


def test_repeated_calls_reuse_workspace(cuda_dev):
    """The workspace carries nothing between calls: a second call on a dirty
    workspace gives the same bits."""
    m, pts, G, x_f32, x_bits, w, sb, sg = make_case("f4_two_row_blocks")
    N, H, W, Cin = x_f32.shape
    Cout = w.shape[0]
    plan = wino.Plan(m, pts, sb, sg, G)
    x = torch.from_numpy(x_bits.view(np.int16).copy()).view(torch.bfloat16).cuda()
    wt = plan.transform_weights(torch.from_numpy(w).cuda())
    ws = torch.full((plan.workspace_bytes(N, H, W, Cin, Cout),), 0x7f, dtype=torch.uint8, device="cuda")
    a = plan.conv2d(x, wt, Cout, out_dtype=torch.float32, workspace=ws).clone()
    b = plan.conv2d(x, wt, Cout, out_dtype=torch.float32, workspace=ws)
    torch.cuda.synchronize()
    assert torch.equal(a, b)


def test_argument_errors_are_status_codes(cuda_dev):
    plan = wino.Plan(4, P4, None, None, 32)
    x = torch.zeros((1, 8, 8, 32), dtype=torch.bfloat16, device="cuda")
    w = torch.zeros((32, 3, 3, 32), dtype=torch.float32, device="cuda")
    wt = plan.transform_weights(w)
    small = torch.empty(16, dtype=torch.uint8, device="cuda")
    with pytest.raises(wino.WinoError) as e:
        plan.conv2d(x, wt, 32, workspace=small)
    assert e.value.status == wino.ERR_WORKSPACE
    with pytest.raises(wino.WinoError) as e:
        plan.conv2d(x, wt, 48)                       # Cout not a multiple of G
    assert e.value.status == wino.ERR_INVALID_ARG
    buf = torch.empty(plan.workspace_bytes(1, 8, 8, 32, 32) + 64, dtype=torch.uint8, device="cuda")
    lib = wino.load_library()
    rc = lib.wino_conv2d_int8(plan._h, x.data_ptr() + 2, wino.BF16, 1, 8, 8, 32, wt.data_ptr(), 32,
                              buf.data_ptr(), wino.F32, buf.data_ptr(), buf.numel(), None)
    assert rc == wino.ERR_INVALID_ARG                # misaligned input pointer
