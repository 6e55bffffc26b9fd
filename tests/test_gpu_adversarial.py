"""GPU parity on inputs built to stress the int8 quantiser Q.

The kernels decide codes with a division-free fast path (t = v * RN(1/s), read
off when every t of a chunk is more than 2^-12 from a half-integer) and fall
back to an fp64 quotient otherwise or when s lies outside [2^-100, 2^100].
Random data reaches the fallback about once in 4000 values; these cases reach
it on purpose and compare every stage with the CPU oracle bit for bit:

* exact ties and near ties in the input transform: an image that is constant
  per channel, transforms with dyadic entries (F(2,3) with identity scales,
  F(4,3) with the textbook Lavin-Gray scales), an anchor channel of value 127
  in every group -- so each (tile, tap, group) scale is |c| * 127 / 127 for the
  tap's integer coefficient c and the other channels divide to exactly their own
  values: half-integers (ties to even), half-integers one ulp either side, and
  +-127 (|v| = absmax);
* extreme scales in the int8-x reading, where Q acts on x itself: a group with
  absmax 1.3 * 2^110 (s above 2^100), one with absmax 1.7 * 2^-110 (s below
  2^-100), one with the denormal absmax 190 * 2^-149 (s = 2^-149, the codes
  clamp at +-127), an all-zero group, and exact ties.
"""
import math

import numpy as np
import pytest
import torch

import oracle
from group_wise_int8_b200 import synth, wino
from tests.gpu_util import assert_bits_equal, rel_l2, run_gpu, run_oracle

pytestmark = pytest.mark.gpu

P2, P4 = synth.POINTS_F2, synth.POINTS_F4
LAVIN_SB = np.array([4, -6, -6, 24, 24, 1], np.float32)
LAVIN_SG = np.array([1 / 4, -1 / 6, -1 / 6, 1 / 24, 1 / 24, 1], np.float32)


def _tie_channels(C, G):
    """Per-channel constants: in each group of G channels an anchor 127 (first group) or -127,
    exact half-integer ties, ties one ulp either side, and the absmax itself."""
    vals = np.zeros(C, np.float32)
    halves = np.array([0.5, 1.5, 2.5, -2.5, -3.5, 62.5, -63.5, 126.5, 4.5, -0.5], np.float32)
    for g in range(C // G):
        blk = np.zeros(G, np.float32)
        blk[g % G] = 127.0 if g % 2 == 0 else -127.0          # the anchor (group absmax)
        k = 0
        for i in range(G):
            if i == g % G:
                continue
            h = halves[k % len(halves)]
            kind = (k // len(halves)) % 4
            if kind == 0:
                blk[i] = h                                    # exact tie
            elif kind == 1:
                blk[i] = np.nextafter(h, np.float32(np.inf))  # one ulp above
            elif kind == 2:
                blk[i] = np.nextafter(h, np.float32(-np.inf))  # one ulp below
            else:
                blk[i] = -blk[g % G] if k % 2 else 100.0      # -absmax, or a plain value
            k += 1
        vals[g * G:(g + 1) * G] = blk
    return vals


@pytest.mark.parametrize("y_path", [wino.YPATH_RECOMPUTE, wino.YPATH_Y32])
@pytest.mark.parametrize("m", [2, 4])
def test_input_transform_ties_and_near_ties(cuda_dev, m, y_path):
    pts, sb, sg = (P2, None, None) if m == 2 else (P4, LAVIN_SB, LAVIN_SG)
    N, H, W, C, Cout, G = 1, 13, 11, 64, 64, 32
    x = np.broadcast_to(_tie_channels(C, G), (N, H, W, C)).astype(np.float32).copy()
    w = synth.make_weights(synth.random_layer(9, m, N, H, W, C, Cout, G, workload="adversarial"))
    ref = run_oracle(m, pts, sb, sg, G, x, w)
    # the construction does reach ties: some transformed values divide to exactly k + 1/2
    Vf = oracle.input_transform(oracle.Plan(m, pts, sb, sg), x, G, want_float=True, quantize=False)[2]
    s = np.repeat(ref["sV"], G, axis=-1).astype(np.float64)
    ratio = np.divide(Vf.astype(np.float64), s, out=np.zeros_like(s), where=s > 0)
    assert np.any((np.abs(ratio) % 1.0) == 0.5)
    got = run_gpu(m, pts, sb, sg, G, x, None, w, out_dtype=torch.float32, y_path=y_path, debug=wino.DEBUG_YQ)
    for k in ("Uq", "sU", "Vq", "sV", "Yq", "sY") + (("Y",) if y_path == wino.YPATH_Y32 else ()):
        assert_bits_equal(k, got[k], ref[k])
    assert_bits_equal("out", got["out"], ref["out"])


def _extreme_x(N, H, W, C, G, seed=3):
    r = np.random.default_rng(seed)
    x = r.standard_normal((N, H, W, C)).astype(np.float32)
    d = np.float32(2.0 ** -149)
    grp = x[0, 0, 0, :G]                       # s above 2^100
    grp[:] = r.uniform(-1, 1, G).astype(np.float32) * np.float32(2.0 ** 110)
    grp[5] = np.float32(1.3 * 2.0 ** 110)
    grp = x[0, 0, 1, :G]                       # s below 2^-100 (normal values)
    grp[:] = r.uniform(-1, 1, G).astype(np.float32) * np.float32(2.0 ** -110)
    grp[7] = np.float32(-1.7 * 2.0 ** -110)
    grp = x[0, 1, 0, :G]                       # denormal absmax: s = 2^-149, codes clamp
    grp[:] = 0.0
    grp[0], grp[1], grp[2], grp[3] = 190 * d, -150 * d, 3 * d, -d
    x[0, 1, 1, :G] = 0.0                       # all-zero group
    grp = x[0, 2, 2, :G]                       # exact ties and near ties at s = 1
    grp[:] = _tie_channels(G, G)
    return x


@pytest.mark.parametrize("y_path", [wino.YPATH_RECOMPUTE, wino.YPATH_Y32])
def test_x_int8_extreme_scales(cuda_dev, y_path):
    m, pts, N, H, W, C, Cout, G = 4, P4, 1, 10, 9, 64, 64, 32
    x = _extreme_x(N, H, W, C, G)
    layer = synth.random_layer(10, m, N, H, W, C, Cout, G, workload="adversarial")
    w = synth.make_weights(layer)
    sb, sg = synth.make_scales(layer)
    xq = oracle.quantize_input(x, G)
    assert xq[0, 1, 0, 0] == np.float32(127 * 2.0 ** -149)    # the clamp acted
    assert xq[0, 1, 0, 1] == np.float32(-127 * 2.0 ** -149)
    ref = run_oracle(m, pts, sb, sg, G, x, w, x_int8=True)
    got = run_gpu(m, pts, sb, sg, G, x, None, w, out_dtype=torch.float32, y_path=y_path, debug=wino.DEBUG_YQ,
                  x_int8=True)
    for k in ("Uq", "sU", "Vq", "sV", "Yq", "sY") + (("Y",) if y_path == wino.YPATH_Y32 else ()):
        assert_bits_equal(k, got[k], ref[k])
    assert_bits_equal("out", got["out"], ref["out"])
    assert np.isfinite(got["out"]).all()
