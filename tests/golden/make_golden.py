"""Write tests/golden/tiny_oracle.json: digests of every stage of the CPU oracle
on the seeded tiny workload (F(4,3), N1 C32 16x16, fp32, identity scales, G=32)
and on a row-norm-balanced F(6,3) variant of it, also under each alternative
reading (per-tap Y groups, int8 x, int8 transforms).

Only the oracle is called.  The fixture freezes the oracle's arithmetic: a later
change to it must regenerate this file and say in its commit message which
passage of the paper's pages (or which reading of it) justifies the change.
Run:  python tests/golden/make_golden.py
"""
import hashlib
import json
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from group_wise_int8_b200 import synth  # noqa: E402


def digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()[:32]


def case(m, balanced, per_tap=False, x_int8=False, int8_transforms=False):
    layer = synth.workload("tiny")[0]
    x, _ = synth.make_input(layer)
    w = synth.make_weights(layer)
    pts = synth.POINTS_F4 if m == 4 else synth.POINTS_F6
    sb = sg = None
    if balanced:
        p0 = oracle.Plan(m, pts)
        sb = (1.0 / np.linalg.norm(p0.BT_d, axis=1)).astype(np.float32)
        sg = (1.0 / np.linalg.norm(p0.G_d, axis=1)).astype(np.float32)
    res = oracle.run_pipeline(oracle.Plan(m, pts, sb, sg, int8_transforms=int8_transforms), x, w, 32,
                              per_tap=per_tap, x_int8=x_int8)
    ref = oracle.conv_direct_f64(x, w)
    out = {k: digest(res[k]) for k in ("Uq", "sU", "Vq", "sV", "Y", "Yq", "sY", "out")}
    out["sqnr_db"] = round(oracle.sqnr_db(ref, res["out"]), 6)
    out["S_B"] = None if sb is None else [float(v) for v in sb]
    out["S_G"] = None if sg is None else [float(v) for v in sg]
    return out


def main():
    data = {
        "what": "oracle stage digests (sha256 prefix of the raw little-endian bytes) and SQNR vs fp64 direct conv",
        "workload": "tiny: N1 C32 16x16 fp32 N(0,1), w ~ N(0,1/(9 Cin)), seed 0, G=32",
        "f4_identity": case(4, False),
        "f6_rownorm": case(6, True),
        # the alternative readings, each alone
        "f6_rownorm_y_tap": case(6, True, per_tap=True),
        "f6_rownorm_x_int8": case(6, True, x_int8=True),
        "f6_rownorm_int8_transforms": case(6, True, int8_transforms=True),
    }
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.json")
    with open(path, "w") as f:
        json.dump(data, f, indent=1)
    print(path)


if __name__ == "__main__":
    main()
