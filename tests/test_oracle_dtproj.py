"""Pins for the oracle of the forward with the dt projection fused (calm-mamba 0.1.4,
"Mamba operator", step 4: dt = dt_proj(dt_low)).  The projection is a library matmul; these
checks fix its wiring against the mixer oracle pinned in test_oracle_pins.py: with W_dt the
identity the fused oracle is the plain one on dt_raw = dt_low; with W_dt a scaled selection
of columns it is the plain one on the selected, scaled columns (both exact in fp64); and on a
tiny case the projection written out as loops matches the matmul.  A transposed W_dt, a
projection over the wrong axis or a dropped term fails one of them.
"""

import numpy as np

from oracle import mixer_oracle as O
from tests.test_oracle_pins import rand_case


def _plain(c, dt_raw):
    return O.mixer(c["xp"], c["z"], dt_raw, c["B"], c["C"], c["A_log"], c["D"], c["conv_w"],
                   c["conv_b"], c["dt_bias"])


def test_identity_projection_is_the_plain_forward():
    c = rand_case(41, Bt=2, L=9, Di=6, N=4)
    W = np.eye(6)
    got = O.mixer_dtproj(c["xp"], c["z"], c["dt_raw"], W, c["B"], c["C"], c["A_log"], c["D"],
                         c["conv_w"], c["conv_b"], c["dt_bias"])
    for g, r in zip(got, _plain(c, c["dt_raw"])):
        np.testing.assert_array_equal(g, r)


def test_column_selection_projection():
    c = rand_case(42, Bt=2, L=7, Di=5, N=3)
    R = 8
    rng = np.random.default_rng(3)
    dt_low = rng.standard_normal((2, 7, R))
    pick = np.array([3, 0, 7, 7, 1])           # channel d takes column pick[d], times 2
    W = np.zeros((5, R))
    W[np.arange(5), pick] = 2.0
    got = O.mixer_dtproj(c["xp"], c["z"], dt_low, W, c["B"], c["C"], c["A_log"], c["D"],
                         c["conv_w"], c["conv_b"], c["dt_bias"])
    for g, r in zip(got, _plain(c, 2.0 * dt_low[:, :, pick])):
        np.testing.assert_array_equal(g, r)


def test_projection_written_out_matches():
    c = rand_case(43, Bt=1, L=5, Di=3, N=2)
    rng = np.random.default_rng(4)
    dt_low = rng.standard_normal((1, 5, 4))
    W = rng.standard_normal((3, 4))
    dt_raw = np.zeros((1, 5, 3))
    for t in range(5):
        for d in range(3):
            for r in range(4):
                dt_raw[0, t, d] += dt_low[0, t, r] * W[d, r]
    got = O.mixer_dtproj(c["xp"], c["z"], dt_low, W, c["B"], c["C"], c["A_log"], c["D"],
                         c["conv_w"], c["conv_b"], c["dt_bias"])
    for g, r in zip(got, _plain(c, dt_raw)):
        np.testing.assert_allclose(g, r, rtol=1e-12, atol=1e-12)


def test_channel_subset_matches_the_whole():
    from selective_state_space_silu_b200 import inputs as I
    w = I.Workload("dtp", 2, 40, 24, 16, 4, "bf16", 4040)
    inp = I.make_dtproj_inputs(w, 16)
    f = I.as_f64
    full = O.mixer_dtproj(f(inp["xp"]), f(inp["z"]), f(inp["dt_low"]), f(inp["W_dt"]), f(inp["B"]),
                          f(inp["C"]), inp["A_log"], inp["D"], inp["conv_w"], inp["conv_b"],
                          inp["dt_bias"])
    di = np.array([0, 5, 23])
    sub = O.mixer_dtproj_channels(inp, np.arange(2), di, widen=f)
    np.testing.assert_allclose(sub[0], full[0][:, :, di], rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(sub[1], full[1][:, di], rtol=1e-13, atol=1e-13)
