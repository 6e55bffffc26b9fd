"""Pins for the CPU oracle: checks against what the paper's pages and the
mathematics fix, not against the oracle itself.

Pins (each chosen so that a plausible slip -- a dropped term, a wrong sign or
index, a transposed operand, a wrong grouping axis -- fails at least one):
  * Winograd identity: with quantisation off the transforms reproduce direct
    3x3 correlation (fp64 to 1e-12; fp32 to 1e-4 for F(4,3), 1e-3 for F(6,3)),
    checked against torch's fp64 conv2d, a library routine.
  * Vandermonde factorisation B^T = S_B V^{-T}, G = S_G V, A^T = V^T S_A with
    S_A S_B S_G = I ("What carries the argument", Sec. 7.1): inverse property
    and scale invariance of the unquantised output.
  * Textbook special case: Lavin & Gray's F(4,3) matrices (the work the pages
    cite as [15]) are a diagonal rescaling of the Vandermonde transforms.
  * Quantiser hand cases (absmax, ties to even, zero group, clamp), and for the
    tile-spanning Y requantisation a hand-written case whose every code and
    scale is fixed (ties that round-half-away would move, a maximum at an odd
    tap, groups that strided couts would split) plus a clamp after a denormal
    scale.
  * Brute-force integer accumulators and the fp32 dequantisation bound.
  * Grouping-axis properties: per-tap V/U groups make the output invariant to
    power-of-two trades between S_B and S_G; tile-spanning Y groups make it
    depend on the per-tap profile of S_A but not on a uniform factor.
"""
import math
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth

P2, P4, P6 = synth.POINTS_F2, synth.POINTS_F4, synth.POINTS_F6


def torch_conv_f64(x, w):
    """Library fp64 3x3 correlation, stride 1, pad 1; x NHWC, w [Cout][3][3][Cin]."""
    xt = torch.from_numpy(np.asarray(x, np.float64)).permute(0, 3, 1, 2)
    wt = torch.from_numpy(np.asarray(w, np.float64)).permute(0, 3, 1, 2)
    return torch.nn.functional.conv2d(xt, wt, padding=1).permute(0, 2, 3, 1).numpy()


def rel_l2(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def rand_case(seed, N=2, H=13, W=11, Cin=8, Cout=5):
    r = np.random.default_rng(seed)
    x = r.standard_normal((N, H, W, Cin)).astype(np.float32)
    w = (r.standard_normal((Cout, 3, 3, Cin)) / math.sqrt(9 * Cin)).astype(np.float32)
    return x, w


def dyadic_scales(seed, n):
    r = np.random.default_rng(seed)
    return (r.integers(32, 129, n) / 64.0).astype(np.float32)


# ---------------------------------------------------------------- plan pins

def _vandermonde_frac(points, b):
    rows = []
    for p in points:
        f, g = (Fraction(1), Fraction(0)) if math.isinf(p) else (Fraction(p), Fraction(1))
        rows.append([f ** j * g ** (b - 1 - j) for j in range(b)])
    return rows


@pytest.mark.parametrize("m,pts", [(2, P2), (4, P4), (6, P6)])
def test_plan_inverse_property(m, pts):
    """B^T V^T = S_B (B^T = S_B V^{-T}); with identity scales B^T V^T = I to rounding."""
    n = m + 2
    sb = dyadic_scales(1, n)
    p = oracle.Plan(m, pts, sb, None)
    V = np.array([[float(v) for v in row] for row in _vandermonde_frac(pts, n)])
    prod = p.BT_d @ V.T
    assert np.allclose(prod, np.diag(sb.astype(np.float64)), atol=1e-12, rtol=0)


def test_lavin_gray_f43_special_case():
    """Lavin & Gray's F(4x4,3x3) matrices, reproduced exactly by S_B, S_G below."""
    BT = np.array([[4, 0, -5, 0, 1, 0], [0, -4, -4, 1, 1, 0], [0, 4, -4, -1, 1, 0],
                   [0, -2, -1, 2, 1, 0], [0, 2, -1, -2, 1, 0], [0, 4, 0, -5, 0, 1]], np.float64)
    G = np.array([[1 / 4, 0, 0], [-1 / 6, -1 / 6, -1 / 6], [-1 / 6, 1 / 6, -1 / 6],
                  [1 / 24, 1 / 12, 1 / 6], [1 / 24, -1 / 12, 1 / 6], [0, 0, 1]], np.float64)
    AT = np.array([[1, 1, 1, 1, 1, 0], [0, 1, -1, 2, -2, 0], [0, 1, 1, 4, 4, 0],
                   [0, 1, -1, 8, -8, 1]], np.float64)
    sb = np.array([4, -6, -6, 24, 24, 1], np.float32)
    sg = np.array([1 / 4, -1 / 6, -1 / 6, 1 / 24, 1 / 24, 1], np.float32)
    p = oracle.Plan(4, P4, sb, sg)
    assert np.array_equal(p.BT_f.astype(np.float64), BT)
    assert np.allclose(p.G_d, G, rtol=1e-7, atol=0)      # S_G entries are fp32 inputs
    assert np.allclose(p.AT_d, AT, rtol=1e-7, atol=0)


def test_textbook_f23_special_case():
    """The textbook F(2x2,3x3) matrices (points 0, 1, -1, inf), reproduced exactly by S_B, S_G below."""
    BT = np.array([[1, 0, -1, 0], [0, 1, 1, 0], [0, -1, 1, 0], [0, 1, 0, -1]], np.float64)
    G = np.array([[1, 0, 0], [0.5, 0.5, 0.5], [0.5, -0.5, 0.5], [0, 0, 1]], np.float64)
    AT = np.array([[1, 1, 1, 0], [0, 1, -1, -1]], np.float64)
    sb = np.array([1, 2, 2, -1], np.float32)
    sg = np.array([1, 0.5, 0.5, 1], np.float32)
    p = oracle.Plan(2, P2, sb, sg)
    assert np.array_equal(p.BT_f.astype(np.float64), BT)
    assert np.array_equal(p.G_d, G)          # dyadic entries: exact
    assert np.array_equal(p.AT_d, AT)


def test_plan_rejects_duplicate_points():
    with pytest.raises(ValueError):
        oracle.Plan(4, (0.0, 1.0, 1.0, 2.0, -2.0, math.inf))


# --------------------------------------------------- Winograd identity (quant off)

@pytest.mark.parametrize("m,pts", [(2, P2), (4, P4), (6, P6)])
@pytest.mark.parametrize("scaled", [False, True])
def test_winograd_identity_f64(m, pts, scaled):
    x, w = rand_case(10 + m)
    n = m + 2
    sb, sg = (dyadic_scales(2, n), dyadic_scales(3, n)) if scaled else (None, None)
    p = oracle.Plan(m, pts, sb, sg)
    ref = torch_conv_f64(x, w)
    assert rel_l2(oracle.conv_wino_f64(p, x, w), ref) < 1e-12


def test_direct_conv_matches_library():
    x, w = rand_case(5, N=1, H=9, W=7, Cin=6, Cout=4)
    assert rel_l2(oracle.conv_direct_f64(x, w), torch_conv_f64(x, w)) < 1e-14


@pytest.mark.parametrize("m,pts,tol", [(4, P4, 1e-4), (6, P6, 1e-3)])
def test_winograd_identity_f32(m, pts, tol):
    x, w = rand_case(20 + m, N=2, H=17, W=14, Cin=16, Cout=8)
    p = oracle.Plan(m, pts)
    err = rel_l2(oracle.conv_wino_f32(p, x, w), torch_conv_f64(x, w))
    assert err < tol
    assert err < 2e-5   # fp32 transforms: far inside the stated bound


@pytest.mark.parametrize("m,pts", [(2, P2), (4, P4), (6, P6)])
def test_scale_invariance_unquantised(m, pts):
    """Any S_B, S_G with S_A = (S_B S_G)^{-1} leaves the unquantised output unchanged."""
    x, w = rand_case(30 + m, N=1, H=12, W=12, Cin=4, Cout=3)
    n = m + 2
    r = np.random.default_rng(7)
    sb = np.exp(r.uniform(np.log(0.5), np.log(2), n)).astype(np.float32)
    sg = np.exp(r.uniform(np.log(0.5), np.log(2), n)).astype(np.float32)
    a = oracle.conv_wino_f64(oracle.Plan(m, pts), x, w)
    b = oracle.conv_wino_f64(oracle.Plan(m, pts, sb, sg), x, w)
    assert rel_l2(b, a) < 1e-12


@pytest.mark.parametrize("mutation", ["transpose_BT", "flip_AT_sign", "drop_G_row", "swap_taps"])
def test_identity_pin_catches_planted_matrix_mistakes(mutation):
    """A mistake planted in the oracle's transform matrices breaks the identity pin."""
    x, w = rand_case(40, N=1, H=8, W=8, Cin=3, Cout=2)
    p = oracle.Plan(4, P4)
    if mutation == "transpose_BT":
        p.BT_d = np.ascontiguousarray(p.BT_d.T)
    elif mutation == "flip_AT_sign":
        p.AT_d = p.AT_d.copy()
        p.AT_d[1, 3] = -p.AT_d[1, 3]
    elif mutation == "drop_G_row":
        p.G_d = p.G_d.copy()
        p.G_d[5, :] = 0
    elif mutation == "swap_taps":
        p.BT_d = np.ascontiguousarray(p.BT_d[[0, 2, 1, 3, 4, 5]])
    assert rel_l2(oracle.conv_wino_f64(p, x, w), torch_conv_f64(x, w)) > 1e-3


# ------------------------------------------------------------ stage pins

@pytest.mark.parametrize("m,pts", [(2, P2), (4, P4), (6, P6)])
def test_input_transform_matches_matmul(m, pts):
    """V = B^T d B per tile and channel (tile origin (ty m - 1, tx m - 1), zero padding)."""
    n = m + 2
    x, _ = rand_case(50, N=1, H=2 * m + 1, W=m + 3, Cin=4)
    p = oracle.Plan(m, pts, dyadic_scales(4, n), None)
    _, _, Vf = oracle.input_transform(p, x, 4, want_float=True, quantize=False)
    H, W = x.shape[1:3]
    TH, TW = -(-H // m), -(-W // m)
    xp = np.zeros((TH * m + 2, TW * m + 2, 4))
    xp[1:H + 1, 1:W + 1] = x[0]
    BT = p.BT_f.astype(np.float64)
    for ty in range(TH):
        for tx in range(TW):
            d = xp[ty * m:ty * m + n, tx * m:tx * m + n]           # [n][n][C]
            ref = np.einsum("ik,klc,jl->ijc", BT, d, BT).reshape(n * n, 4)
            got = Vf[ty * TW + tx]
            bound = 8 * n * np.finfo(np.float32).eps * np.einsum(
                "ik,klc,jl->ijc", abs(BT), abs(d), abs(BT)).reshape(n * n, 4) + 1e-30
            assert np.all(np.abs(got - ref) <= bound)


@pytest.mark.parametrize("m,pts", [(2, P2), (4, P4), (6, P6)])
def test_weight_transform_matches_matmul(m, pts):
    n = m + 2
    _, w = rand_case(60, Cin=8, Cout=3)
    p = oracle.Plan(m, pts, None, dyadic_scales(5, n))
    Uq, sU, Uf = oracle.weight_transform(p, w, 8, want_float=True)
    ref = np.einsum("ia,oabc,jb->ijoc", p.G_d, w.astype(np.float64), p.G_d).reshape(n * n, 3, 8)
    assert np.allclose(Uf, ref, rtol=2 ** -23, atol=1e-30)
    # dequantised codes are within half a step of the fp32 value
    s_full = np.repeat(sU, 8, axis=-1).astype(np.float64)
    assert np.all(np.abs(Uq * s_full - Uf) <= 0.5 * s_full * (1 + 1e-6) + 1e-30)


QUANT_CASES = [
    # values, expected codes, expected scale
    ([127.0, -63.5, 0.5, 1.5, 2.5, -0.5], [127, -64, 0, 2, 2, 0], 1.0),
    ([254.0, 1.0, 3.0, -5.0], [127, 0, 2, -2], 2.0),            # 0.5 -> 0, 1.5 -> 2, -2.5 -> -2
    ([0.0, -0.0, 0.0], [0, 0, 0], 0.0),                          # zero group
    ([-3.0], [-127], np.float32(3.0) / np.float32(127.0)),
    ([1.0, 0.25], [127, 32], np.float32(1.0) / np.float32(127.0)),  # 0.25 / (1/127) = 31.75 -> 32
]


@pytest.mark.parametrize("vals,codes,scale", QUANT_CASES)
def test_quantiser_hand_cases(vals, codes, scale):
    q, s = oracle.quantize(np.array(vals, np.float32))
    assert list(q) == codes
    assert np.float32(s) == np.float32(scale)


def test_quantiser_range_and_error():
    r = np.random.default_rng(3)
    for _ in range(200):
        v = (r.standard_normal(64) * 10 ** r.uniform(-3, 3)).astype(np.float32)
        q, s = oracle.quantize(v)
        assert q.min() >= -127 and q.max() <= 127
        assert np.max(np.abs(q)) == 127                           # absmax maps to +-127
        assert np.all(np.abs(q * np.float64(s) - v) <= 0.5 * s * (1 + 1e-5))


@pytest.mark.parametrize("G", [8, 16])
def test_int32_accumulators_brute_force(G):
    r = np.random.default_rng(8)
    n2, T, Cin, Cout = 9, 7, 3 * G, 5
    Vq = r.integers(-127, 128, (T, n2, Cin)).astype(np.int8)
    Uq = r.integers(-127, 128, (n2, Cout, Cin)).astype(np.int8)
    sV = r.uniform(0.01, 2, (T, n2, Cin // G)).astype(np.float32)
    sU = r.uniform(0.01, 2, (n2, Cout, Cin // G)).astype(np.float32)
    Y, acc = oracle.hadamard(n2, Vq, sV, Uq, sU, G, want_acc=True)
    ref = np.einsum("tpgc,pogc->ptog", Vq.astype(np.int64).reshape(T, n2, -1, G),
                    Uq.astype(np.int64).reshape(n2, Cout, -1, G))
    assert np.array_equal(acc.astype(np.int64), ref)
    # Y = sum_j acc_j sV_j sU_j up to fp32 rounding of the chain
    terms = ref.transpose(1, 0, 2, 3) * (sV[:, :, None, :].astype(np.float64) * sU[None].astype(np.float64))
    exact = terms.sum(-1)
    bound = (Cin // G + 2) * np.finfo(np.float32).eps * np.abs(terms).sum(-1) + 1e-30
    assert np.all(np.abs(Y - exact) <= bound)


def test_output_transform_matches_matmul():
    m, n = 4, 6
    p = oracle.Plan(m, P4, dyadic_scales(9, n), dyadic_scales(10, n))
    r = np.random.default_rng(11)
    N, H, W, Cout, G = 1, 7, 5, 4, 2
    T = N * 2 * 2
    Yq = r.integers(-127, 128, (T, n * n, Cout)).astype(np.int8)
    sY = r.uniform(0.1, 1, (T, Cout // G)).astype(np.float32)
    out = oracle.output_transform(p, Yq, sY, N, H, W, G)
    AT = p.AT_f.astype(np.float64)
    for t in range(T):
        ty, tx = divmod(t, 2)
        for co in range(Cout):
            Yd = (np.float32(sY[t, co // G]) * Yq[t, :, co].astype(np.float32)).astype(np.float64).reshape(n, n)
            ref = AT @ Yd @ AT.T
            bound = 4 * n * np.finfo(np.float32).eps * (abs(AT) @ abs(Yd) @ abs(AT).T)
            for i in range(m):
                for j in range(m):
                    yy, xx = ty * m + i, tx * m + j
                    if yy < H and xx < W:
                        assert abs(out[0, yy, xx, co] - ref[i, j]) <= bound[i, j] + 1e-30


# ------------------------------------------------------ grouping properties

def _pipeline_out(m, pts, sb, sg, x, w, G):
    return oracle.run_pipeline(oracle.Plan(m, pts, sb, sg), x, w, G)


def test_power_of_two_trade_between_SB_SG_is_exact():
    """Per-tap V and U groups absorb any per-tap power of two moved from S_G to S_B."""
    m, n, G = 6, 8, 16
    x, w = rand_case(70, N=1, H=12, W=12, Cin=32, Cout=32)
    sb, sg = dyadic_scales(12, n), dyadic_scales(13, n)
    k = np.random.default_rng(14).integers(-2, 3, n).astype(np.float32)
    a = _pipeline_out(m, P6, sb, sg, x, w, G)
    b = _pipeline_out(m, P6, sb * 2.0 ** k, sg * 2.0 ** -k, x, w, G)
    assert np.array_equal(a["Vq"], b["Vq"]) and np.array_equal(a["Uq"], b["Uq"])
    assert np.array_equal(a["Yq"], b["Yq"]) and np.array_equal(a["out"], b["out"])


def test_y_groups_span_taps():
    """A uniform power-of-two factor on S_A is absorbed exactly; a per-tap profile is not.

    If Y were grouped per tap, any per-tap power of two would be absorbed too.
    """
    m, n, G = 6, 8, 16
    x, w = rand_case(71, N=1, H=12, W=12, Cin=32, Cout=32)
    sb, sg = dyadic_scales(15, n), dyadic_scales(16, n)
    base = _pipeline_out(m, P6, sb, sg, x, w, G)
    uni = _pipeline_out(m, P6, sb * 2.0, sg, x, w, G)
    assert np.array_equal(base["out"], uni["out"])
    k = np.array([0, 1, -1, 2, 0, -2, 1, 0], np.float32)
    prof = _pipeline_out(m, P6, sb * 2.0 ** k, sg, x, w, G)
    assert np.array_equal(base["Vq"], prof["Vq"])           # V groups are per tap
    assert not np.array_equal(base["Yq"], prof["Yq"])       # Y groups span taps
    ref = oracle.conv_direct_f64(x, w)
    assert abs(oracle.sqnr_db(ref, base["out"]) - oracle.sqnr_db(ref, prof["out"])) > 0.1


@pytest.mark.parametrize("m,pts", [(4, P4), (6, P6)])
def test_y_tap_reading_absorbs_per_tap_powers_of_two(m, pts):
    """The per-tap Y reading (Y_TAP): a per-tap power-of-two profile on S_B scales
    V, Y and sY of each tap (i, j) by d_i d_j exactly and A^T's column xi by 1/d_xi,
    so the per-tap groups give bit-identical codes and output.  With the default
    tile-spanning groups the same profile changes the codes (test_y_groups_span_taps)."""
    n, G = m + 2, 16
    x, w = rand_case(72, N=1, H=13, W=11, Cin=32, Cout=32)
    sb, sg = dyadic_scales(17, n), dyadic_scales(18, n)
    k = np.array([0, 1, -1, 2, 0, -2, 1, 0][:n], np.float32)
    base = oracle.run_pipeline(oracle.Plan(m, pts, sb, sg), x, w, G, per_tap=True)
    prof = oracle.run_pipeline(oracle.Plan(m, pts, sb * 2.0 ** k, sg), x, w, G, per_tap=True)
    assert np.array_equal(base["Vq"], prof["Vq"]) and np.array_equal(base["Yq"], prof["Yq"])
    d = 2.0 ** k.astype(np.float64)
    ratio = (d[:, None] * d[None, :]).reshape(-1)                # tap (i, j) -> d_i d_j
    assert np.array_equal(prof["sY"].astype(np.float64), base["sY"].astype(np.float64) * ratio[None, :, None])
    assert np.array_equal(base["out"], prof["out"])


def test_y_tap_scales_are_per_tap_group_maxima():
    """sY[t][tap][j] = max |Y[t][tap][jG:(j+1)G]| / 127 (IEEE division), codes = rne(Y / sY)."""
    r = np.random.default_rng(5)
    T, n2, Cout, G = 3, 16, 64, 32
    Y = (r.standard_normal((T, n2, Cout)) * np.exp(r.standard_normal((T, n2, 1)))).astype(np.float32)
    Y[1, 3, :G] = 0.0                                              # an all-zero group
    Yq, sY = oracle.y_requant(n2, Y, G, per_tap=True)
    amax = np.abs(Y.reshape(T, n2, Cout // G, G)).max(axis=-1)
    assert np.array_equal(sY, (amax / np.float32(127.0)).astype(np.float32))
    assert sY[1, 3, 0] == 0.0 and not Yq[1, 3, :G].any()
    assert np.abs(Yq.astype(np.int32)).max() == 127
    q = Yq.reshape(T, n2, Cout // G, G).astype(np.float64) * sY[..., None]
    err = np.abs(q - Y.reshape(T, n2, Cout // G, G))
    assert np.all(err <= 0.5 * sY[..., None] * (1 + 1e-6) + 1e-30)


# -------------------------------------- Y requantisation, tile-spanning groups
# The default reading: one scale per (tile, G consecutive output channels) over
# all n*n taps of the tile (review, "Core claim" and Fig. 3: Y's cross-shaped
# per-tap spread is what the group must span), Q with s = absmax/127 and ties to
# even.  The hand case below fixes every code and scale by hand; each entry
# names the slip it catches.

_DENORM = 2.0 ** -149          # the smallest positive fp32 (a denormal)


def _y_hand_case():
    """T = 2 tiles, n2 = 16 taps (F(2,3)), Cout = 4, G = 2 (groups {0,1} and {2,3})."""
    T, n2, Cout = 2, 16, 4
    Y = np.zeros((T, n2, Cout), np.float32)
    Yq = np.zeros((T, n2, Cout), np.int8)
    sY = np.zeros((T, 2), np.float32)

    def put(t, tap, co, v, q):
        Y[t, tap, co] = v
        Yq[t, tap, co] = q

    # tile 0, group 0: the maximum 127 sits at an odd tap (13), so s = 1 exactly; a maximum taken
    # over even taps only would give s = 100.25/127 and different codes
    put(0, 13, 1, -127.0, -127)
    put(0, 0, 0, 100.25, 100)
    put(0, 2, 0, 0.5, 0)            # tie: to even 0 (half away from zero: 1)
    put(0, 5, 0, 1.5, 2)            # tie: 2 either way
    put(0, 6, 1, 2.5, 2)            # tie: to even 2 (half away: 3)
    put(0, 7, 1, -2.5, -2)          # tie: to even -2 (half away: -3)
    put(0, 8, 0, -3.5, -4)          # tie: to even -4
    sY[0, 0] = 1.0
    # tile 0, group 1 (couts 2, 3): all zero -> s = 0, every code 0
    # tile 1, group 0: maximum 63.5 at tap 3 -> s = 0.5 exactly
    put(1, 3, 0, 63.5, 127)
    put(1, 4, 1, 0.25, 0)           # 0.5 -> 0 (half away: 1)
    put(1, 9, 1, 0.75, 2)           # 1.5 -> 2
    put(1, 10, 0, -31.25, -62)      # -62.5 -> -62 (half away: -63)
    sY[1, 0] = 0.5
    # tile 1, group 1: maximum |-254| at tap 15, cout 3 -> s = 2 exactly.  With groups of strided
    # couts ({0, 2}, {1, 3}) tile 0's group of couts {0, 2} would get s = 100.25/127.
    put(1, 15, 3, -254.0, -127)
    put(1, 1, 2, 5.0, 2)            # 2.5 -> 2 (half away: 3)
    put(1, 14, 2, 254.0, 127)
    put(1, 12, 3, 3.0, 2)           # 1.5 -> 2
    sY[1, 1] = 2.0
    return Y, Yq, sY


def test_y_tile_requant_hand_case():
    Y, want_q, want_s = _y_hand_case()
    Yq, sY = oracle.y_requant(16, Y, 2)
    assert sY.shape == (2, 2)
    assert np.array_equal(sY, want_s)
    assert np.array_equal(Yq, want_q)


def test_y_tile_requant_clamps_after_a_denormal_scale():
    """absmax = 190 * 2^-149 (a denormal): s = RN(190/127 * 2^-149) = 2^-149, so 190 * 2^-149
    divides to 190 and is clamped to 127 (and -150 * 2^-149 to -127); 3 * 2^-149 stays 3."""
    Y = np.zeros((1, 4, 2), np.float32)
    Y[0, 1, 0] = np.float32(190 * _DENORM)
    Y[0, 2, 1] = np.float32(-150 * _DENORM)
    Y[0, 3, 1] = np.float32(3 * _DENORM)
    Yq, sY = oracle.y_requant(4, Y, 2)
    assert sY[0, 0] == np.float32(_DENORM)
    assert Yq[0, 1, 0] == 127 and Yq[0, 2, 1] == -127 and Yq[0, 3, 1] == 3
    assert np.count_nonzero(Yq) == 3


@pytest.mark.parametrize("n2,G", [(36, 32), (64, 64)])
def test_y_tile_scales_are_maxima_over_every_tap_and_group_channel(n2, G):
    """sY[t][j] = RN(max over all n2 taps and the G couts j*G..j*G+G-1 of |Y| / 127).  Every
    group's maximum is planted at a random tap (odd taps included) and a random cout of the
    group, with the rest of the group well below it, so a partial span of taps or couts, or
    another grouping of the couts, changes the scale."""
    r = np.random.default_rng(41)
    T, Cout = 5, 4 * G
    Y = (r.standard_normal((T, n2, Cout)) * 0.25).astype(np.float32)
    Y[:, :, :G] = 0.0
    Y[2, :, G:2 * G] = 0.0                       # one all-zero group
    peak_tap = np.zeros((T, Cout // G), int)
    for t in range(T):
        for j in range(Cout // G):
            if (t == 2 and j == 1) or j == 0:
                continue
            tap, co = int(r.integers(n2)), j * G + int(r.integers(G))
            peak_tap[t, j] = tap
            Y[t, tap, co] = np.float32((1 if r.random() < 0.5 else -1) * (3.0 + r.random()))
    Y[:, 5, 3] = np.float32(2.0)                 # group 0: maxima at odd tap 5 only
    Yq, sY = oracle.y_requant(n2, Y, G)
    amax = np.abs(Y).reshape(T, n2, Cout // G, G).max(axis=(1, 3))
    assert np.array_equal(sY, amax / np.float32(127.0))
    assert np.all(sY[:, 0] == np.float32(2.0) / np.float32(127.0))
    assert sY[2, 1] == 0.0 and not Yq[2, :, G:2 * G].any()
    assert np.any(peak_tap % 2 == 1)
    q = Yq.reshape(T, n2, Cout // G, G).astype(np.float64)
    s = sY[:, None, :, None].astype(np.float64)
    assert np.all(np.abs(q * s - Y.reshape(T, n2, Cout // G, G)) <= 0.5 * s * (1 + 1e-6) + 1e-45)
    # the planted maxima map to +-127
    for t in range(T):
        for j in range(1, Cout // G):
            if sY[t, j] > 0:
                assert np.abs(Yq[t, :, j * G:(j + 1) * G].astype(int)).max() == 127


def test_output_transform_tap_matches_matmul():
    """Per-tap reading: out = A^T Yd A with Yd[xi][nu] = sY[t][xi*n+nu][co/G] * Yq, within the
    fp32 rounding bound of the two fma chains.  The scales differ by powers of two from tap to
    tap, so using the scale of another tap (a transposed tap index, a single scale per tile)
    breaks the bound."""
    m, n = 4, 6
    p = oracle.Plan(m, P4, dyadic_scales(19, n), dyadic_scales(20, n))
    r = np.random.default_rng(21)
    N, H, W, Cout, G = 1, 7, 6, 4, 2
    T = N * 2 * 2
    n2 = n * n
    Yq = r.integers(-127, 128, (T, n2, Cout)).astype(np.int8)
    sY = (r.uniform(0.5, 1, (T, n2, Cout // G)) * 2.0 ** r.integers(-6, 7, (T, n2, Cout // G))).astype(np.float32)
    out = oracle.output_transform(p, Yq, sY, N, H, W, G, per_tap=True)
    AT = p.AT_f.astype(np.float64)
    for t in range(T):
        ty, tx = divmod(t, 2)
        for co in range(Cout):
            Yd = (sY[t, :, co // G] * Yq[t, :, co].astype(np.float32)).astype(np.float64).reshape(n, n)
            ref = AT @ Yd @ AT.T
            bound = 4 * n * np.finfo(np.float32).eps * (abs(AT) @ abs(Yd) @ abs(AT).T)
            for i in range(m):
                for j in range(m):
                    yy, xx = ty * m + i, tx * m + j
                    if yy < H and xx < W:
                        assert abs(out[0, yy, xx, co] - ref[i, j]) <= bound[i, j] + 1e-30


@pytest.mark.parametrize("m,pts", [(4, P4), (6, P6)])
def test_standard_scales_collapse_and_row_norm_scales_recover(m, pts):
    """The pages: with standard scales fully quantized Winograd collapses (FID > 300),
    and rescaling the rows of B^T and G (their row norms) removes Y's per-tap
    imbalance.  Under the tile-spanning Y groups the quantised output with
    identity scales has negative SQNR, and row-norm balancing scales recover it."""
    layer = synth.workload("tiny")[0]
    x, _ = synth.make_input(layer)
    w = synth.make_weights(layer)
    ref = oracle.conv_direct_f64(x, w)
    p0 = oracle.Plan(m, pts)
    sb = (1.0 / np.linalg.norm(p0.BT_d, axis=1)).astype(np.float32)
    sg = (1.0 / np.linalg.norm(p0.G_d, axis=1)).astype(np.float32)
    s_std = oracle.sqnr_db(ref, oracle.run_pipeline(p0, x, w, 32)["out"])
    s_bal = oracle.sqnr_db(ref, oracle.run_pipeline(oracle.Plan(m, pts, sb, sg), x, w, 32)["out"])
    assert s_std < 0.0
    assert s_bal > 10.0
    assert s_bal > s_std + 20.0


# ------------------------------------------- alternative input-side readings
# Eqs. (14)-(16) give the quantised input transform the scales "sqB sqB sqx": an
# int8 B^T (one scale per matrix, applied on both sides) and an int8 x.  The
# library offers both as plan options (x_int8, int8_transforms); these pins fix
# the oracle's side of them.

def _exact_code(v, amax):
    """rne(127 v / amax) in exact rationals, clamped to +-127, and whether it sits within
    1e-4 of a tie (where the fp32 division may decide either way)."""
    t = Fraction(float(v)) * 127 / Fraction(float(amax))
    frac = t - math.floor(t)
    return max(-127, min(127, round(t))), abs(frac - Fraction(1, 2)) < Fraction(1, 10 ** 4)


def _check_int8_matrix(got, exact):
    """got = s * q entrywise with s = max|exact| / 127 (fp32) and q the exact-rational
    rne codes of exact (either neighbour at a tie)."""
    amax = float(np.abs(exact).max())
    s = np.float32(amax) / np.float32(127.0)
    for v, g in zip(np.asarray(exact, np.float64).ravel(), np.asarray(got).ravel()):
        q, tie = _exact_code(v, amax)
        want = {np.float32(s * np.float32(c)) for c in ((q - 1, q, q + 1) if tie else (q,))}
        assert np.float32(g) in want, (v, g, q, want)


def test_int8_transforms_lavin_gray_codes():
    """Int8 transforms on the Lavin-Gray F(4,3) matrices: B^T's largest entry is 5, so its
    codes are rne(127 v / 5) (4 -> 102, 1 -> 25, 2 -> 51, -5 -> -127); A^T's is 8 (1 -> 16,
    2 -> 32, 8 -> 127; 4 lands on the tie 63.5, decided by the fp32 division)."""
    sb = np.array([4, -6, -6, 24, 24, 1], np.float32)
    sg = np.array([1 / 4, -1 / 6, -1 / 6, 1 / 24, 1 / 24, 1], np.float32)
    BT = np.array([[4, 0, -5, 0, 1, 0], [0, -4, -4, 1, 1, 0], [0, 4, -4, -1, 1, 0],
                   [0, -2, -1, 2, 1, 0], [0, 2, -1, -2, 1, 0], [0, 4, 0, -5, 0, 1]], np.float64)
    AT = np.array([[1, 1, 1, 1, 1, 0], [0, 1, -1, 2, -2, 0], [0, 1, 1, 4, 4, 0],
                   [0, 1, -1, 8, -8, 1]], np.float64)
    p = oracle.Plan(4, P4, sb, sg, int8_transforms=True)
    exact = oracle.Plan(4, P4, sb, sg)
    assert _exact_code(4, 5) == (102, False) and _exact_code(4, 8) == (64, True)
    _check_int8_matrix(p.BT_f, BT)
    _check_int8_matrix(p.AT_f, exact.AT_d)        # A^T = AT up to the fp32 scales S_A
    assert np.array_equal(p.G_d, exact.G_d) and np.array_equal(p.BT_d, exact.BT_d)
    s = np.float32(5.0) / np.float32(127.0)
    assert p.BT_f[0, 0] == np.float32(s * np.float32(102)) and p.BT_f[0, 2] == -np.float32(s * np.float32(127))


@pytest.mark.parametrize("m,pts", [(4, P4), (6, P6)])
def test_int8_transforms_error_bound_and_zeros(m, pts):
    """Every entry moves by at most half a step of its matrix's scale, zeros stay zero, the
    largest entry maps to +-127 steps, and no entry exceeds 127 steps."""
    n = m + 2
    sb, sg = dyadic_scales(31, n), dyadic_scales(32, n)
    p = oracle.Plan(m, pts, sb, sg, int8_transforms=True)
    exact = oracle.Plan(m, pts, sb, sg)
    for got, ref in ((p.BT_f, exact.BT_f), (p.AT_f, exact.AT_f)):
        s = float(np.float32(np.abs(ref).max()) / np.float32(127.0))
        err = np.abs(got.astype(np.float64) - ref.astype(np.float64))
        assert np.all(err <= 0.5 * s * (1 + 1e-5))
        assert np.all(got[ref == 0] == 0)
        codes = got.astype(np.float64) / s
        assert np.allclose(codes, np.round(codes), rtol=0, atol=1e-4) and np.abs(codes).max() <= 127 + 1e-4
        assert abs(abs(codes.ravel()[np.argmax(np.abs(ref))]) - 127) < 1e-4


def test_int8_transforms_change_nothing_on_the_int8_grid():
    """The textbook F(2,3) matrices hold only 0 and +-1, so each becomes 127 steps of 1/127:
    in fp32 (1/127) * 127 rounds back to 1, the plan is unchanged and so is every stage."""
    sb = np.array([1, 2, 2, -1], np.float32)
    sg = np.array([1, 0.5, 0.5, 1], np.float32)
    p0, p1 = oracle.Plan(2, P2, sb, sg), oracle.Plan(2, P2, sb, sg, int8_transforms=True)
    assert np.array_equal(p0.BT_f, p1.BT_f) and np.array_equal(p0.AT_f, p1.AT_f)
    x, w = rand_case(81, N=1, H=9, W=10, Cin=32, Cout=32)
    a, b = oracle.run_pipeline(p0, x, w, 32), oracle.run_pipeline(p1, x, w, 32)
    for k in ("Vq", "sV", "Yq", "sY", "out"):
        assert np.array_equal(a[k], b[k])


def test_x_int8_codes_per_pixel_group_brute_force():
    """x through Q per pixel and G consecutive channels: s = absmax / 127 of that group
    only (fp32 division) and codes rne(127 x / absmax) in exact rationals (either neighbour
    at a tie); an outlier in one group leaves every other group untouched."""
    r = np.random.default_rng(9)
    G = 16
    x = (r.standard_normal((2, 3, 2, 48)) * np.exp(r.standard_normal((2, 3, 2, 3)).repeat(G, axis=-1)))
    x = x.astype(np.float32)
    x[1, 2, 0, G:2 * G] = 0.0                                   # an all-zero group
    xq = oracle.quantize_input(x, G)
    assert not xq[1, 2, 0, G:2 * G].any()
    for idx in np.ndindex(*x.shape[:3]):
        for j in range(3):
            grp, got = x[idx][j * G:(j + 1) * G], xq[idx][j * G:(j + 1) * G]
            if not grp.any():
                continue
            _check_int8_matrix(got, grp.astype(np.float64))
    y = x.copy()
    y[0, 1, 1, 5] = 1e4                                          # outlier in group 0 of one pixel
    yq = oracle.quantize_input(y, G)
    changed = np.argwhere(np.any((yq != xq).reshape(2, 3, 2, 3, G), axis=-1))
    assert changed.tolist() == [[0, 1, 1, 0]]


def test_x_int8_changes_nothing_on_the_int8_grid():
    """Values k / 8 with integer |k| <= 127 and a +-127 in every group are their own codes
    (s = 1/8 exactly): the quantised input equals x and the whole pipeline is unchanged."""
    r = np.random.default_rng(10)
    N, H, W, C, G = 1, 11, 9, 64, 32
    k = r.integers(-127, 128, (N, H, W, C))
    k[..., 0], k[..., G] = 127, -127
    x = (k / 8.0).astype(np.float32)
    assert np.array_equal(oracle.quantize_input(x, G), x)
    w = (r.standard_normal((32, 3, 3, C)) / 24).astype(np.float32)
    p = oracle.Plan(4, P4, dyadic_scales(3, 6), dyadic_scales(4, 6))
    a, b = oracle.run_pipeline(p, x, w, G), oracle.run_pipeline(p, x, w, G, x_int8=True)
    for key in ("Vq", "sV", "Yq", "sY", "out"):
        assert np.array_equal(a[key], b[key])
