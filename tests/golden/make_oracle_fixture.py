"""Writes oracle_toy.json: the fp64 oracle's results on a tiny seeded case (the toy workload shrunk
to 2 sender heads, 3 receiver heads and 256 tokens).

The pages print no worked example, so no value here comes from them.  The fixture pins the
oracle to itself over time: a change to its arithmetic shows up as a failing comparison, and the
commit that makes it must name the passage (or the reading of it) that justifies it.  Only the
oracle and the input generator are called.

    python tests/golden/make_oracle_fixture.py
"""
import json
import os
import sys

import numpy as np

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from cross_model_attention_mr_b200.workloads import config, draw_layers, shrink  # noqa: E402

SPEC = dict(L=256, H_s=2, H_r=3)
ROWS = [0, 1, 63, 64, 127, 200, 255]


def compute():
    spec = shrink(config(1), **SPEC)
    lay = draw_layers(spec)[0]
    p = float(np.float32(spec.p))
    r = oracle.compress(lay.Q, lay.K, spec.scale, p, spec.block, lay.bias, n_threads=1)
    O = oracle.retrieve_rows(lay.Q, lay.K, spec.scale, spec.block, r.kept, lay.W, lay.V, np.asarray(ROWS),
                             lay.bias, n_threads=1)
    return {
        "case": {"workload": "toy_L512_d64_f32 shrunk", **SPEC, "p": p, "block": spec.block, "rows": ROWS},
        "kept": r.kept.astype(int).tolist(),
        "count": r.count.astype(int).tolist(),
        "mass": r.mass.tolist(),
        "kept_mass": r.kept_mass.tolist(),
        "lse": r.lse.tolist(),
        "O_rows": O.tolist(),
    }


if __name__ == "__main__":
    oracle.build()
    with open(os.path.join(HERE, "oracle_toy.json"), "w") as f:
        json.dump(compute(), f)
    print("wrote", os.path.join(HERE, "oracle_toy.json"))
