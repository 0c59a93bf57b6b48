"""Writes tests/golden/ssd_tiny_oracle_samples.json: outputs of the Mamba2 oracle (scan,
conv + SiLU over x|B|C, gated RMSNorm) on the seeded ssd_tiny workload at fixed sample
positions, in fp64.

A regression fixture for the oracle itself: the pages print no worked example for the
Mamba2 layer, so the values come from the oracle (this script calls only oracle/ and the
seeded input generator).  Regenerate only when a change to the oracle's arithmetic is
justified by the pages, and say which passage in the commit.

    python tests/golden/make_golden_ssd.py
"""

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(os.path.dirname(HERE))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

from oracle import ssd_oracle as so  # noqa: E402
from selective_state_space_silu_b200 import inputs as I  # noqa: E402

OUT = os.path.join(HERE, "ssd_tiny_oracle_samples.json")
Y_SAMPLES = [(0, 0, 0, 0), (0, 99, 3, 63), (1, 50, 2, 17), (1, 7, 1, 40), (0, 64, 0, 5)]
H_SAMPLES = [(0, 0, 0, 0), (1, 3, 63, 63), (0, 2, 10, 33)]


def inputs():
    d = I.make_ssd_inputs(I.SSD_WORKLOADS["ssd_tiny"])
    r = np.random.default_rng(77)
    Cc = 4 * 64 + 2 * 64
    xbc = I.f32_to_bf16_bits(r.standard_normal((2, 20, Cc)).astype(np.float32))
    conv_w = r.uniform(-0.5, 0.5, size=(Cc, 4)).astype(np.float32)
    ids = np.array([[0] * 12 + [1] * 8, [5] * 20])
    nw = r.standard_normal(256).astype(np.float32)
    return d, xbc, conv_w, ids, nw


def compute():
    d, xbc, conv_w, ids, nw = inputs()
    y, h = so.ssd(d["x"], d["dt_raw"], d["A_log"], d["B"], d["C"], d["D"], d["dt_bias"], z=d["z"])
    conv, cs = so.conv_silu(xbc, conv_w, seq_idx=ids)
    norm = so.gated_rmsnorm(d["x"].reshape(2, 100, 256), d["z"].reshape(2, 100, 256), nw)
    return {
        "workload": "ssd_tiny (batch 2, L 100, 4 heads x 64, d_state 64, gate, seed 2000); "
                    "conv: 2 x 20 x 384 channels, seed 77; norm over the ssd_tiny x and z",
        "y": [[list(ix), float(y[ix])] for ix in Y_SAMPLES],
        "h_out": [[list(ix), float(h[ix])] for ix in H_SAMPLES],
        "conv": [[[0, 11, 5], float(conv[0, 11, 5])], [[0, 12, 300], float(conv[0, 12, 300])],
                 [[1, 19, 383], float(conv[1, 19, 383])]],
        "conv_state_out_b0_c7": [float(v) for v in cs[0, 7]],
        "norm": [[[0, 0, 0], float(norm[0, 0, 0])], [[1, 99, 255], float(norm[1, 99, 255])]],
    }


if __name__ == "__main__":
    with open(OUT, "w") as f:
        json.dump(compute(), f, indent=1)
    print(OUT)
