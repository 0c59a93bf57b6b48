"""Pins for the backward oracle (oracle_mixer_bwd_f64): every gradient against central
finite differences of the forward oracle (pinned by test_oracle_pins.py) -- an
independent route, so a dropped chain-rule term, a wrong sign or a wrong index in the
backward fails here -- plus the special cases that fix whole gradients to zero."""

import numpy as np
import pytest

from tests.test_oracle_pins import rand_case, run

GRAD_OF = {"dxp": "xp", "dz": "z", "ddt_raw": "dt_raw", "dB": "B", "dC": "C",
           "dA_log": "A_log", "dD": "D", "dconv_w": "conv_w", "dconv_b": "conv_b",
           "ddt_bias": "dt_bias"}


def loss(oracle, c, dy):
    y, _, _ = run(oracle, c)
    return float((y * dy).sum())


def bwd(oracle, c, dy):
    return oracle.mixer_bwd(c["xp"], c["z"], c["dt_raw"], c["B"], c["C"], c["A_log"], c["D"],
                            c["conv_w"], c["conv_b"], c["dt_bias"], dy)


@pytest.mark.parametrize("seed,N,conv_b", [(11, 3, True), (12, 4, False), (13, 2, True)])
def test_every_gradient_matches_finite_differences(oracle, seed, N, conv_b):
    c = rand_case(seed, Bt=2, L=7, Di=3, N=N, conv_b=conv_b, A_range=(-1.0, 1.5))
    dy = np.random.default_rng(seed + 100).standard_normal(c["xp"].shape)
    g = bwd(oracle, c, dy)
    eps = 1e-6
    for gname, name in GRAD_OF.items():
        if c[name] is None:
            assert g[gname] is None
            continue
        fd = np.zeros_like(c[name])
        for ix in np.ndindex(c[name].shape):
            cp = {k: (None if v is None else np.array(v, dtype=np.float64)) for k, v in c.items()}
            cp[name][ix] += eps
            lp = loss(oracle, cp, dy)
            cp[name][ix] -= 2 * eps
            lm = loss(oracle, cp, dy)
            fd[ix] = (lp - lm) / (2 * eps)
        err = np.abs(fd - g[gname]) / (1.0 + np.abs(fd))
        assert err.max() < 2e-6, (gname, err.max())


def test_zero_upstream_gradient_gives_zeros(oracle):
    c = rand_case(20, Bt=1, L=5, Di=2, N=3)
    g = bwd(oracle, c, np.zeros(c["xp"].shape))
    for k, v in g.items():
        assert v is None or not np.any(v), k


def test_zero_B_leaves_no_state_gradients(oracle):
    """B = 0: the state stays 0, so C and A_log get no gradient (B itself does)."""
    c = rand_case(21, Bt=2, L=6, Di=2, N=3)
    c["B"] = np.zeros_like(c["B"])
    dy = np.random.default_rng(5).standard_normal(c["xp"].shape)
    g = bwd(oracle, c, dy)
    assert not np.any(g["dC"]) and not np.any(g["dA_log"])
    assert np.any(g["dB"])


@pytest.mark.parametrize("case", ["length_one_docs", "consecutive_boundaries", "many_short_docs"])
def test_packed_and_cached_gradients_match_finite_differences(oracle, case):
    """With documents (seq_idx) and a cached start (h_in, conv_state_in): every gradient,
    the two state gradients included, against central differences of the forward oracle."""
    from selective_state_space_silu_b200 import inputs as I
    c = rand_case(30 + len(case), Bt=2, L=9, Di=2, N=3, state=True, A_range=(-1.0, 1.5))
    seq = I.seq_idx_case(case, 2, 9, edge=4, seed=3)
    dy = np.random.default_rng(77).standard_normal(c["xp"].shape)
    g = oracle.mixer_bwd(c["xp"], c["z"], c["dt_raw"], c["B"], c["C"], c["A_log"], c["D"],
                         c["conv_w"], c["conv_b"], c["dt_bias"], dy, seq_idx=seq,
                         h_in=c["h_in"], conv_state_in=c["conv_state_in"])

    def loss_of(cc):
        y, _, _ = run(oracle, cc, seq_idx=seq)
        return float((y * dy).sum())

    eps = 1e-6
    names = dict(GRAD_OF, dh_in="h_in", dconv_state_in="conv_state_in")
    for gname, name in names.items():
        fd = np.zeros_like(c[name])
        for ix in np.ndindex(c[name].shape):
            cp = {k: (None if v is None else np.array(v, dtype=np.float64)) for k, v in c.items()}
            cp[name][ix] += eps
            lp = loss_of(cp)
            cp[name][ix] -= 2 * eps
            lm = loss_of(cp)
            fd[ix] = (lp - lm) / (2 * eps)
        err = np.abs(fd - g[gname]) / (1.0 + np.abs(fd))
        assert err.max() < 2e-6, (case, gname, err.max())
