"""Pins for the CPU oracle: checks against things other than the oracle itself.

Every check here uses an independent route to the answer -- a closed form, a library
routine (numpy.convolve, numpy.logaddexp, scipy.special.expit, numpy.cumsum), or the
recurrence unrolled as an explicit O(L^2) sum -- so that a plausible mistake in the
oracle (a dropped term, a wrong sign, a wrong tap order, a transposed operand, a wrong
conv-state orientation) fails at least one of them.

The operator is calm-mamba 0.1.4 (PKG-INFO, section "Mamba operator"), steps 2 and 4-6;
the decode contract (prefill-then-step equals a full forward) is niverel-mamba 0.1.0,
section "Autoregressive decoding"; the kill-selectivity control is the Octopus Research
report, section 1.
"""

import numpy as np
import pytest
from scipy.special import expit

from tests.tolerances import assert_close, same_nonfinite_pattern, within


# ---------------------------------------------------------------- independent pieces
def np_silu(v):
    return v * expit(v)


def np_softplus(v):
    return np.logaddexp(0.0, v)


def np_conv_u(xp_bd, w_d, b_d, state_d=None):
    """u[t] for one channel via numpy.convolve over the left-padded sequence."""
    K = w_d.shape[0]
    pad = np.zeros(K - 1) if state_d is None else np.asarray(state_d, dtype=np.float64)
    xpad = np.concatenate([pad, xp_bd])
    pre = np.convolve(xpad, w_d[::-1], mode="valid") + (0.0 if b_d is None else b_d)
    return np_silu(pre), xpad


def rand_case(seed, Bt=2, L=8, Di=3, N=3, K=4, conv_b=True, state=False, A_range=(-1, 2)):
    r = np.random.default_rng(seed)
    c = dict(
        xp=r.standard_normal((Bt, L, Di)),
        z=r.standard_normal((Bt, L, Di)),
        dt_raw=0.5 * r.standard_normal((Bt, L, Di)),
        B=r.standard_normal((Bt, L, N)),
        C=r.standard_normal((Bt, L, N)),
        A_log=r.uniform(*A_range, size=(Di, N)),
        D=r.standard_normal(Di),
        conv_w=r.uniform(-0.5, 0.5, size=(Di, K)),
        conv_b=r.uniform(-0.5, 0.5, size=Di) if conv_b else None,
        dt_bias=r.uniform(-4.0, -1.0, size=Di),
        h_in=r.standard_normal((Bt, Di, N)) if state else None,
        conv_state_in=r.standard_normal((Bt, Di, K - 1)) if state else None,
    )
    return c


def run(oracle, c, **kw):
    return oracle.mixer(c["xp"], c["z"], c["dt_raw"], c["B"], c["C"], c["A_log"], c["D"],
                        c["conv_w"], c["conv_b"], c["dt_bias"], c.get("h_in"),
                        c.get("conv_state_in"), **kw)


def brute_force(c):
    """The recurrence unrolled as an explicit sum over source steps s <= t:

    h_t[n] = exp(A_n * sum_{r<=t} Delta_r) h0[n]
             + sum_{s<=t} exp(A_n * sum_{s<r<=t} Delta_r) * Delta_s * B_s[n] * u_s
    """
    xp, z, dtr, Bm, Cm = c["xp"], c["z"], c["dt_raw"], c["B"], c["C"]
    Bt, L, Di = xp.shape
    N = Bm.shape[2]
    K = c["conv_w"].shape[1]
    A = -np.exp(c["A_log"])
    y = np.zeros((Bt, L, Di))
    hT = np.zeros((Bt, Di, N))
    cs = np.zeros((Bt, Di, K - 1))
    for b in range(Bt):
        for d in range(Di):
            st = None if c.get("conv_state_in") is None else c["conv_state_in"][b, d]
            u, xpad = np_conv_u(xp[b, :, d], c["conv_w"][d],
                                None if c["conv_b"] is None else c["conv_b"][d], st)
            delta = np_softplus(dtr[b, :, d] + c["dt_bias"][d])
            h0 = np.zeros(N) if c.get("h_in") is None else c["h_in"][b, d]
            for t in range(L):
                h = np.exp(A[d] * delta[: t + 1].sum()) * h0
                for s in range(t + 1):
                    h = h + np.exp(A[d] * delta[s + 1: t + 1].sum()) * delta[s] * Bm[b, s] * u[s]
                y[b, t, d] = (Cm[b, t] @ h + c["D"][d] * u[t]) * np_silu(z[b, t, d])
                if t == L - 1:
                    hT[b, d] = h
            cs[b, d] = xpad[L:]
    return y, hT, cs


# ---------------------------------------------------------------- P1: explicit sum
@pytest.mark.parametrize("seed,state,conv_b", [(1, False, True), (2, True, True), (3, False, False),
                                               (4, True, False)])
def test_p1_matches_unrolled_sum(oracle, seed, state, conv_b):
    c = rand_case(seed, Bt=2, L=8, Di=2, N=3, state=state, conv_b=conv_b)
    y, h, cs = run(oracle, c)
    yb, hb, csb = brute_force(c)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h, hb, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cs, csb)


def test_p1_other_conv_width(oracle):
    c = rand_case(11, Bt=1, L=7, Di=2, N=2, K=2, state=True)
    y, h, cs = run(oracle, c)
    yb, hb, csb = brute_force(c)
    np.testing.assert_allclose(y, yb, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(h, hb, rtol=1e-12, atol=1e-13)
    np.testing.assert_array_equal(cs, csb)


# ---------------------------------------------------------------- P2: geometric series
def test_p2_geometric_closed_form(oracle):
    Bt, L, Di, N = 1, 40, 2, 4
    xc, dtc, zc = 0.7, -0.3, 0.9
    Bv = np.array([0.5, -1.0, 2.0, 0.25])
    Cv = np.array([1.5, 0.3, -0.7, 2.0])
    A_log = np.log(np.array([[1.0, 2.0, 3.0, 4.0], [0.5, 1.5, 2.5, 8.0]]))
    c = dict(
        xp=np.full((Bt, L, Di), xc), z=np.full((Bt, L, Di), zc),
        dt_raw=np.full((Bt, L, Di), dtc),
        B=np.tile(Bv, (Bt, L, 1)), C=np.tile(Cv, (Bt, L, 1)),
        A_log=A_log, D=np.array([1.0, -0.5]),
        conv_w=np.tile([0.0, 0.0, 0.0, 1.0], (Di, 1)), conv_b=np.zeros(Di),
        dt_bias=np.array([-1.0, -2.5]),
    )
    y, h, cs = run(oracle, c)
    t = np.arange(L)
    for d in range(Di):
        u = np_silu(xc)                       # conv_w picks the current input only
        delta = np_softplus(dtc + c["dt_bias"][d])
        a = np.exp(delta * -np.exp(A_log[d]))  # per-state decay
        # h_t = Delta*B*u * (1 - a^(t+1)) / (1 - a)   (t zero-based)
        ht = delta * Bv[None, :] * u * (1 - a[None, :] ** (t[:, None] + 1)) / (1 - a[None, :])
        yt = (ht @ Cv + c["D"][d] * u) * np_silu(zc)
        np.testing.assert_allclose(y[0, :, d], yt, rtol=1e-12)
        np.testing.assert_allclose(h[0, d], ht[-1], rtol=1e-12)
    np.testing.assert_array_equal(cs, np.full((Bt, Di, 3), xc))


# ---------------------------------------------------------------- P3: B = 0
def test_p3_zero_B_gives_skip_path_only(oracle):
    c = rand_case(5, Bt=2, L=13, Di=4, N=5)
    c["B"] = np.zeros_like(c["B"])
    y, h, cs = run(oracle, c)
    assert np.all(h == 0.0)
    for b in range(2):
        for d in range(4):
            u, _ = np_conv_u(c["xp"][b, :, d], c["conv_w"][d], c["conv_b"][d])
            np.testing.assert_allclose(y[b, :, d], c["D"][d] * u * np_silu(c["z"][b, :, d]),
                                       rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- P4: L = 1
def test_p4_single_step_closed_form(oracle):
    c = rand_case(6, Bt=3, L=1, Di=4, N=3)
    y, h, cs = run(oracle, c)
    for b in range(3):
        for d in range(4):
            x0 = c["xp"][b, 0, d]
            u = np_silu(c["conv_b"][d] + c["conv_w"][d, 3] * x0)
            delta = np_softplus(c["dt_raw"][b, 0, d] + c["dt_bias"][d])
            hh = delta * c["B"][b, 0] * u
            np.testing.assert_allclose(h[b, d], hh, rtol=1e-13)
            yy = (c["C"][b, 0] @ hh + c["D"][d] * u) * np_silu(c["z"][b, 0, d])
            np.testing.assert_allclose(y[b, 0, d], yy, rtol=1e-13)
            np.testing.assert_array_equal(cs[b, d], [0.0, 0.0, x0])


# ---------------------------------------------------------------- P5: prefill then step
@pytest.mark.parametrize("k", [1, 3, 7])
def test_p5_prefill_then_steps_equals_forward(oracle, k):
    c = rand_case(7, Bt=2, L=12, Di=3, N=4)
    y, h, cs = run(oracle, c)
    L = 12
    pre = {**c}
    for key in ("xp", "z", "dt_raw", "B", "C"):
        pre[key] = c[key][:, : L - k]
    yp, hp, csp = run(oracle, pre)
    ys = [yp]
    for t in range(L - k, L):
        st = {**c, "h_in": hp, "conv_state_in": csp}
        for key in ("xp", "z", "dt_raw", "B", "C"):
            st[key] = c[key][:, t: t + 1]
        yt, hp, csp = run(oracle, st)
        ys.append(yt)
    np.testing.assert_allclose(np.concatenate(ys, axis=1), y, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(hp, h, rtol=1e-13, atol=1e-15)
    np.testing.assert_array_equal(csp, cs)


def test_p5_steps_from_zero_equal_forward(oracle):
    c = rand_case(8, Bt=1, L=6, Di=2, N=3)
    y, h, cs = run(oracle, c)
    hp = np.zeros_like(h)
    csp = np.zeros_like(cs)
    for t in range(6):
        st = {**c, "h_in": hp, "conv_state_in": csp}
        for key in ("xp", "z", "dt_raw", "B", "C"):
            st[key] = c[key][:, t: t + 1]
        yt, hp, csp = run(oracle, st)
        np.testing.assert_allclose(yt[:, 0], y[:, t], rtol=1e-13, atol=1e-15)


# ---------------------------------------------------------------- P6: kill selectivity
def test_p6_kill_selectivity_changes_outputs(oracle):
    c = rand_case(9, Bt=2, L=32, Di=8, N=4)
    y, _, _ = run(oracle, c)
    k = {**c}
    for key in ("dt_raw", "B", "C"):
        k[key] = np.repeat(c[key][:, :1], 32, axis=1)    # time-constant: value at t = 0
    yk, _, _ = run(oracle, k)
    np.testing.assert_allclose(yk[:, 0], y[:, 0], rtol=1e-13)   # t = 0 is unchanged
    frac_outside = 1.0 - within(yk[:, 1:], y[:, 1:], "bf16").mean()
    assert frac_outside > 0.5, frac_outside


# ---------------------------------------------------------------- P7: no decay
def test_p7_no_decay_is_prefix_sum(oracle):
    c = rand_case(10, Bt=2, L=20, Di=3, N=4)
    c["A_log"] = np.full_like(c["A_log"], -200.0)   # A = -1.4e-87: exp(Delta*A) == 1.0
    y, h, _ = run(oracle, c)
    for b in range(2):
        for d in range(3):
            u, _ = np_conv_u(c["xp"][b, :, d], c["conv_w"][d], c["conv_b"][d])
            delta = np_softplus(c["dt_raw"][b, :, d] + c["dt_bias"][d])
            ht = np.cumsum(delta[:, None] * c["B"][b] * u[:, None], axis=0)
            yt = ((ht * c["C"][b]).sum(1) + c["D"][d] * u) * np_silu(c["z"][b, :, d])
            np.testing.assert_allclose(y[b, :, d], yt, rtol=1e-11, atol=1e-13)
            np.testing.assert_allclose(h[b, d], ht[-1], rtol=1e-11, atol=1e-13)


# ---------------------------------------------------------------- P8: full decay
def test_p8_full_decay_is_memoryless(oracle):
    c = rand_case(12, Bt=2, L=9, Di=3, N=5, state=True)
    c["A_log"] = np.full_like(c["A_log"], 20.0)     # A = -4.9e8: exp(Delta*A) == 0.0
    y, h, _ = run(oracle, c)
    for b in range(2):
        for d in range(3):
            st = c["conv_state_in"][b, d]
            u, _ = np_conv_u(c["xp"][b, :, d], c["conv_w"][d], c["conv_b"][d], st)
            delta = np_softplus(c["dt_raw"][b, :, d] + c["dt_bias"][d])
            cb = (c["C"][b] * c["B"][b]).sum(1)
            yt = (delta * u * cb + c["D"][d] * u) * np_silu(c["z"][b, :, d])
            np.testing.assert_allclose(y[b, :, d], yt, rtol=1e-12, atol=1e-14)
            np.testing.assert_allclose(h[b, d], delta[-1] * c["B"][b, -1] * u[-1], rtol=1e-13)


# ---------------------------------------------------------------- P9: invariants
def test_p9_causality(oracle):
    c = rand_case(13, Bt=1, L=16, Di=3, N=4)
    y, _, _ = run(oracle, c)
    for key in ("xp", "dt_raw", "B", "C", "z"):
        p = {**c, key: c[key].copy()}
        p[key][:, 9] += 1.5
        yp, _, _ = run(oracle, p)
        np.testing.assert_array_equal(yp[:, :9], y[:, :9])
        assert np.any(yp[:, 9:] != y[:, 9:])


def test_p9_batch_and_channel_permutation(oracle):
    c = rand_case(14, Bt=3, L=10, Di=5, N=3, state=True)
    y, h, cs = run(oracle, c)
    pb = np.array([2, 0, 1])
    pd = np.array([3, 1, 4, 0, 2])
    p = {**c}
    for key in ("xp", "z", "dt_raw"):
        p[key] = c[key][pb][:, :, pd]
    for key in ("B", "C"):
        p[key] = c[key][pb]
    for key in ("A_log", "D", "conv_w", "conv_b", "dt_bias"):
        p[key] = c[key][pd]
    p["h_in"] = c["h_in"][pb][:, pd]
    p["conv_state_in"] = c["conv_state_in"][pb][:, pd]
    yp, hp, csp = run(oracle, p)
    np.testing.assert_array_equal(yp, y[pb][:, :, pd])
    np.testing.assert_array_equal(hp, h[pb][:, pd])
    np.testing.assert_array_equal(csp, cs[pb][:, pd])


def test_p9_affine_in_B(oracle):
    c = rand_case(15, Bt=2, L=11, Di=3, N=4)
    outs = {}
    for alpha in (0.0, 1.0, 3.7):
        p = {**c, "B": c["B"] * alpha}
        outs[alpha] = run(oracle, p)
    y0, y1, ya = outs[0.0][0], outs[1.0][0], outs[3.7][0]
    np.testing.assert_allclose(ya, y0 + 3.7 * (y1 - y0), rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(outs[3.7][1], 3.7 * outs[1.0][1], rtol=1e-12, atol=1e-14)


@pytest.mark.parametrize("L", [0, 1, 2, 3, 5])
def test_p9_conv_state_out_orientation(oracle, L):
    c = rand_case(16, Bt=2, L=L, Di=3, N=2, state=True)
    _, h, cs = run(oracle, c)
    for b in range(2):
        for d in range(3):
            xpad = np.concatenate([c["conv_state_in"][b, d], c["xp"][b, :, d]])
            np.testing.assert_array_equal(cs[b, d], xpad[-3:])
    if L == 0:   # an empty sequence passes the state through unchanged
        np.testing.assert_array_equal(h, c["h_in"])


# ---------------------------------------------------------------- precision band
@pytest.mark.parametrize("name", ["tiny", "stress"])
def test_fp32_recurrence_sits_inside_fp32_band(oracle, name):
    """A plain fp32 evaluation of the same loops lies inside the fp32 tolerance of fp64."""
    from selective_state_space_silu_b200 import inputs as I
    w = I.WORKLOADS[name]
    d = I.make_inputs(w)
    args = [d[k] for k in ("xp", "z", "dt_raw", "B", "C", "A_log", "D", "conv_w", "conv_b",
                           "dt_bias")]
    y64, h64, _ = oracle.mixer(*args, precision="f64")
    y32, h32, _ = oracle.mixer(*args, precision="f32")
    assert_close(y32, y64, "f32", "y fp32 oracle vs fp64")
    assert_close(h32, h64, "f32", "h fp32 oracle vs fp64")


def test_nonfinite_inputs_propagate(oracle):
    c = rand_case(17, Bt=1, L=6, Di=2, N=2)
    c["xp"][0, 2, 1] = np.nan
    y, h, _ = run(oracle, c)
    assert np.all(np.isfinite(y[0, :2, 1])) and np.all(np.isnan(y[0, 2:, 1]))
    assert np.all(np.isfinite(y[:, :, 0]))
    assert np.all(np.isnan(h[0, 1]))


def test_tolerance_rule_counts_nonfinite_as_mismatch():
    assert not within(np.array([np.nan]), np.array([1.0]), "f32")[0]
    assert not within(np.array([np.nan]), np.array([np.nan]), "f32")[0]
    assert not within(np.array([np.inf]), np.array([np.inf]), "f32")[0]
    fin = same_nonfinite_pattern(np.array([np.nan, np.inf, 1.0]), np.array([np.nan, np.inf, 2.0]))
    assert fin.tolist() == [False, False, True]
    with pytest.raises(AssertionError):
        same_nonfinite_pattern(np.array([np.nan, 1.0]), np.array([1.0, 1.0]))
    with pytest.raises(AssertionError):
        same_nonfinite_pattern(np.array([np.inf]), np.array([-np.inf]))
    assert within(np.array([1.0 + 9e-4]), np.array([1.0]), "f32")[0]
    assert not within(np.array([1.0 + 1.2e-3]), np.array([1.0]), "f32")[0]


# ---------------------------------------------------------------- regression fixture
def test_oracle_matches_its_golden_fixture(oracle):
    """tests/golden/tiny_oracle_samples.json (written by tests/golden/make_golden.py from
    the oracle): any later change to the oracle's arithmetic shows up here."""
    import json
    import os
    from selective_state_space_silu_b200 import inputs as I
    g = json.load(open(os.path.join(os.path.dirname(__file__), "golden",
                                    "tiny_oracle_samples.json")))
    d = I.make_inputs(I.WORKLOADS["tiny"])
    y, h, cs = oracle.mixer(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                            d["conv_w"], d["conv_b"], d["dt_bias"])
    for ix, v in g["y"]:
        assert y[tuple(ix)] == v
    for ix, v in g["h_out"]:
        assert h[tuple(ix)] == v
    assert list(cs[1, 127]) == g["conv_state_out_b1_d127"]
