"""Writes tests/golden/tiny_oracle_samples.json: oracle outputs of the tiny workload
(batch 2, L 16, d_inner 128, d_state 16, fp32) at fixed sample positions, in fp64.

A regression fixture for the oracle itself: the pages print no worked example for this
operator, so the values come from the oracle (this script calls only oracle/ and the seeded
input generator).  Regenerate only when a change to the oracle's arithmetic is justified by
the pages, and say which passage in the commit.

    python tests/golden/make_golden.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from oracle import mixer_oracle as O  # noqa: E402
from selective_state_space_silu_b200 import inputs as I  # noqa: E402

OUT = os.path.join(HERE, "tiny_oracle_samples.json")
Y_SAMPLES = [(0, 0, 0), (0, 15, 127), (1, 7, 64), (1, 3, 5), (0, 9, 100), (1, 15, 0)]
H_SAMPLES = [(0, 0, 0), (1, 127, 15), (0, 64, 7), (1, 5, 3)]


def compute():
    w = I.WORKLOADS["tiny"]
    d = I.make_inputs(w)
    y, h, cs = O.mixer(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                       d["conv_w"], d["conv_b"], d["dt_bias"])
    return {
        "workload": "tiny (batch 2, L 16, d_inner 128, d_state 16, fp32 I/O, seed 1000)",
        "y": [[list(ix), float(y[ix])] for ix in Y_SAMPLES],
        "h_out": [[list(ix), float(h[ix])] for ix in H_SAMPLES],
        "conv_state_out_b1_d127": [float(v) for v in cs[1, 127]],
    }


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(compute(), f, indent=1)
    print(OUT)
