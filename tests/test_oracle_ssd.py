"""Pins for the Mamba2 (SSD) oracle: each check reaches the answer by another route.

* an O(L^2) unrolled sum over source steps (every output as an explicit weighted sum of
  the inputs, including the initial state and document resets);
* the chunked evaluation -- within a chunk a masked (C B^T) matrix with the decay
  exp(cs_t - cs_s) from a cumulative sum, between chunks the carried state -- which the
  pages compare against the sequential oracle (niverel-mamba 0.1.0, section "Measured
  tolerances": chunked vs sequential agree to fp64 rounding);
* closed forms: A -> 0 (a plain numpy.cumsum), A -> -inf (memoryless), constant inputs
  (geometric series), a single step;
* invariants: linearity in (x, h_in), causality, the head -> group mapping, and the
  strict reset (niverel-mamba 0.1.0, section "seq_idx strict reset": a packed row equals
  its documents run one by one).

A dropped term, a wrong sign of A, a swapped B/C, a transposed state, a wrong group
mapping or a missed reset each fail at least one of these.

The layer's conv + SiLU over x, B, C is pinned against numpy.convolve with
scipy.special.expit, the conv-state orientation for L = 0..5, and a packed row against its
documents run alone; the gated RMSNorm against unit mean square per row or group, scale
invariance, the separate-group identity and the gate's direction.
"""

import numpy as np
import pytest
from scipy.special import expit

from oracle import ssd_oracle as so

TOL = 1e-12


def close(a, b, tol=TOL):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    scale = max(1.0, float(np.max(np.abs(b))) if b.size else 1.0)
    err = float(np.max(np.abs(a - b))) if a.size else 0.0
    assert err <= tol * scale, f"max abs err {err:.3e} > {tol:.1e} * {scale:.3g}"


def softplus(v):
    return np.logaddexp(0.0, v)


def silu(v):
    return v * expit(v)


def case(seed, Bt=2, L=9, H=4, P=3, N=5, G=2, z=True, h_in=True, A_range=(-1.0, 1.5)):
    r = np.random.default_rng(seed)
    return dict(
        x=r.standard_normal((Bt, L, H, P)),
        dt_raw=0.5 * r.standard_normal((Bt, L, H)),
        A_log=r.uniform(*A_range, size=H),
        B=r.standard_normal((Bt, L, G, N)),
        C=r.standard_normal((Bt, L, G, N)),
        D=r.standard_normal(H),
        dt_bias=r.uniform(-3.0, 0.0, size=H),
        z=r.standard_normal((Bt, L, H, P)) if z else None,
        h_in=r.standard_normal((Bt, H, P, N)) if h_in else None,
    )


def run(c, **kw):
    return so.ssd(c["x"], c["dt_raw"], c["A_log"], c["B"], c["C"], c["D"], c["dt_bias"],
                  z=c.get("z"), h_in=c.get("h_in"), **kw)


def unrolled(c, seq_idx=None):
    """y_t = sum over s <= t in t's document of (C_t . B_s) exp(A sum_{s<r<=t} Delta_r)
    Delta_s x_s + C_t . (exp(A sum_{r<=t} Delta_r) h_in) (only while no reset has happened)
    + D x_t, times SiLU(z_t); h_out likewise at t = L - 1.  Plain loops."""
    x, dtr, Bm, Cm = c["x"], c["dt_raw"], c["B"], c["C"]
    Bt, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.zeros((Bt, L, H, P))
    hT = np.zeros((Bt, H, P, N))
    for b in range(Bt):
        ids = np.zeros(L, dtype=np.int64) if seq_idx is None else np.asarray(seq_idx)[b]
        for h in range(H):
            g = h // (H // G)
            A = -np.exp(c["A_log"][h])
            dl = softplus(dtr[b, :, h] + c["dt_bias"][h])
            for t in range(L + 1):
                tt = min(t, L - 1)
                acc = np.zeros((P, N))
                for s in range(tt + 1):
                    if ids[s] != ids[tt] or np.any(ids[s:tt + 1] != ids[tt]):
                        continue
                    w = np.exp(A * dl[s + 1:tt + 1].sum()) * dl[s]
                    acc += w * np.outer(x[b, s, h], Bm[b, s, g])
                if c.get("h_in") is not None and np.all(ids[:tt + 1] == ids[0]):
                    acc += np.exp(A * dl[:tt + 1].sum()) * c["h_in"][b, h]
                if t == L:
                    hT[b, h] = acc
                    continue
                yt = acc @ Cm[b, t, g] + c["D"][h] * x[b, t, h]
                if c.get("z") is not None:
                    yt = yt * silu(c["z"][b, t, h])
                y[b, t, h] = yt
    return y, hT


def chunked(c, Q):
    """The chunked form: per chunk, Y = (L o C B^T) (Delta x) + exp(cs) C H^T + D x with
    L[t, s] = exp(cs_t - cs_s) for s <= t (cs the in-chunk cumulative sum of Delta A); the
    carried state H <- exp(cs_last) H + sum_s exp(cs_last - cs_s) Delta_s x_s B_s^T."""
    x, dtr, Bm, Cm = c["x"], c["dt_raw"], c["B"], c["C"]
    Bt, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.zeros((Bt, L, H, P))
    hT = np.zeros((Bt, H, P, N))
    for b in range(Bt):
        for h in range(H):
            g = h // (H // G)
            A = -np.exp(c["A_log"][h])
            Hs = np.zeros((P, N)) if c.get("h_in") is None else c["h_in"][b, h].copy()
            for c0 in range(0, L, Q):
                sl = slice(c0, min(L, c0 + Q))
                dl = softplus(dtr[b, sl, h] + c["dt_bias"][h])
                cs = np.cumsum(dl * A)
                seg = cs[:, None] - cs[None, :]
                Lm = np.where(np.tril(np.ones_like(seg)) > 0, np.exp(np.minimum(seg, 0.0)), 0.0)
                Xd = x[b, sl, h] * dl[:, None]                       # [q, P]
                CB = Cm[b, sl, g] @ Bm[b, sl, g].T                   # [q, q]
                Y = (Lm * CB) @ Xd + np.exp(cs)[:, None] * (Cm[b, sl, g] @ Hs.T) \
                    + c["D"][h] * x[b, sl, h]
                if c.get("z") is not None:
                    Y = Y * silu(c["z"][b, sl, h])
                y[b, sl, h] = Y
                wlast = np.exp(cs[-1] - cs)                          # [q]
                Hs = np.exp(cs[-1]) * Hs + (Xd * wlast[:, None]).T @ Bm[b, sl, g]
            hT[b, h] = Hs
    return y, hT


def test_unrolled_sum():
    for seed in range(3):
        c = case(10 + seed)
        y, hT = run(c)
        yu, hu = unrolled(c)
        close(y, yu)
        close(hT, hu)


def test_unrolled_sum_with_resets():
    c = case(20, L=11)
    ids = np.array([[0, 0, 0, 1, 1, 2, 2, 2, 2, 3, 3],
                    [5, 6, 6, 6, 6, 6, 7, 8, 8, 8, 8]])
    y, hT = run(c, seq_idx=ids)
    yu, hu = unrolled(c, seq_idx=ids)
    close(y, yu)
    close(hT, hu)


@pytest.mark.parametrize("Q,L", [(4, 13), (8, 8), (3, 10), (16, 5)])
def test_chunked_form(Q, L):
    c = case(30 + Q, L=L, H=3, G=1, N=6)
    y, hT = run(c)
    yc, hc = chunked(c, Q)
    close(y, yc)
    close(hT, hc)


def test_a_to_zero_is_cumsum():
    # A_log = -200: A = -e^-200, exp(Delta A) == 1 exactly, so h is a running sum
    c = case(40, z=False, h_in=False, G=1)
    c["A_log"][:] = -200.0
    y, hT = run(c)
    dl = softplus(c["dt_raw"] + c["dt_bias"])                          # [Bt, L, H]
    inc = (dl[..., None] * c["x"])[..., None] * c["B"][:, :, 0][:, :, None, None, :]
    hs = np.cumsum(inc, axis=1)                                          # [Bt, L, H, P, N]
    close(hT, hs[:, -1])
    yy = np.einsum("blhpn,bln->blhp", hs, c["C"][:, :, 0]) + c["D"][None, None, :, None] * c["x"]
    close(y, yy)


def test_a_to_minus_inf_is_memoryless():
    # A_log = 20: exp(Delta A) underflows to 0, so only the current step contributes
    c = case(50, z=False, h_in=True, G=1)
    c["A_log"][:] = 20.0
    y, hT = run(c)
    dl = softplus(c["dt_raw"] + c["dt_bias"])
    cb = np.einsum("bln,bln->bl", c["C"][:, :, 0], c["B"][:, :, 0])
    yy = (dl * cb[..., None])[..., None] * c["x"] + c["D"][None, None, :, None] * c["x"]
    close(y, yy)
    close(hT, (dl[:, -1, :, None] * c["x"][:, -1])[..., None] * c["B"][:, -1, 0][:, None, None, :])


def test_constant_inputs_geometric():
    # constant Delta, x, B, C: h_t = Delta x B (1 - a^(t+1)) / (1 - a), a = exp(Delta A)
    Bt, L, H, P, N = 1, 12, 2, 2, 3
    c = case(60, Bt=Bt, L=L, H=H, P=P, N=N, G=1, z=False, h_in=False)
    r = np.random.default_rng(61)
    x0, B0, C0 = r.standard_normal((H, P)), r.standard_normal(N), r.standard_normal(N)
    c["x"][:] = x0[None, None]
    c["B"][:] = B0
    c["C"][:] = C0
    c["dt_raw"][:] = 0.3
    y, hT = run(c)
    dl = softplus(0.3 + c["dt_bias"])
    a = np.exp(-dl * np.exp(c["A_log"]))
    for t in range(L):
        geo = (1 - a ** (t + 1)) / (1 - a)                               # [H]
        ht = (dl * geo)[:, None, None] * x0[:, :, None] * B0[None, None, :]
        close(y[0, t], ht @ C0 + c["D"][:, None] * x0)
    close(hT[0], ht)


def test_single_step():
    c = case(70, L=1, G=2)
    y, hT = run(c)
    dl = softplus(c["dt_raw"][:, 0] + c["dt_bias"])                     # [Bt, H]
    a = np.exp(-dl * np.exp(c["A_log"]))
    grp = np.arange(4) // 2
    Bg, Cg = c["B"][:, 0][:, grp], c["C"][:, 0][:, grp]                  # [Bt, H, N]
    h1 = a[..., None, None] * c["h_in"] + (dl[..., None] * c["x"][:, 0])[..., None] * Bg[:, :, None, :]
    close(hT, h1)
    yy = np.einsum("bhpn,bhn->bhp", h1, Cg) + c["D"][None, :, None] * c["x"][:, 0]
    close(y[:, 0], yy * silu(c["z"][:, 0]))


def test_linear_in_x_and_state():
    c = case(80, z=False)
    y1, h1 = run(c)
    c2 = dict(c, x=2.5 * c["x"], h_in=2.5 * c["h_in"])
    y2, h2 = run(c2)
    close(y2, 2.5 * y1)
    close(h2, 2.5 * h1)


def test_causal():
    c = case(90, L=10)
    y1, _ = run(c)
    c2 = {k: (v.copy() if isinstance(v, np.ndarray) else v) for k, v in c.items()}
    t0 = 6
    for k in ("x", "dt_raw", "B", "C", "z"):
        c2[k][:, t0] += 1.0
    y2, _ = run(c2)
    assert np.array_equal(y1[:, :t0], y2[:, :t0])
    assert np.max(np.abs(y1[:, t0] - y2[:, t0])) > 1e-3


def test_group_mapping():
    # G = 2 over H = 4: heads 0-1 read group 0, heads 2-3 group 1
    c = case(100, G=2)
    y, hT = run(c)
    for g in range(2):
        hs = slice(2 * g, 2 * g + 2)
        sub = dict(x=c["x"][:, :, hs], dt_raw=c["dt_raw"][:, :, hs], A_log=c["A_log"][hs],
                   B=c["B"][:, :, g:g + 1], C=c["C"][:, :, g:g + 1], D=c["D"][hs],
                   dt_bias=c["dt_bias"][hs], z=c["z"][:, :, hs], h_in=c["h_in"][:, hs])
        ys, hs_ = run(sub)
        close(y[:, :, hs], ys)
        close(hT[:, hs], hs_)


def test_packed_row_equals_documents():
    c = case(110, Bt=1, L=12, h_in=False)
    ids = np.array([[3, 3, 3, 3, 9, 9, 4, 4, 4, 4, 4, 4]])
    y, hT = run(c, seq_idx=ids)
    for lo, hi in ((0, 4), (4, 6), (6, 12)):
        sub = dict(c, x=c["x"][:, lo:hi], dt_raw=c["dt_raw"][:, lo:hi], B=c["B"][:, lo:hi],
                   C=c["C"][:, lo:hi], z=c["z"][:, lo:hi])
        ys, hs = run(sub)
        close(y[:, lo:hi], ys)
    close(hT, hs)


def test_bf16_bits_read_exactly():
    c = case(120, z=True)
    bits = {k: (np.ascontiguousarray(c[k], dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)
            for k in ("x", "dt_raw", "B", "C", "z")}
    widened = {k: (v.astype(np.uint32) << 16).view(np.float32).astype(np.float64) for k, v in bits.items()}
    y1, h1 = run(dict(c, **bits))
    y2, h2 = run(dict(c, **widened))
    assert np.array_equal(y1, y2) and np.array_equal(h1, h2)


def test_channel_subset():
    c = case(130, Bt=2, H=4, G=2)
    y, hT = run(c)
    sel = [(0, 1), (1, 3), (1, 0)]
    outs, hs = so.ssd_channels(c["x"], c["dt_raw"], c["A_log"], c["B"], c["C"], c["D"],
                               c["dt_bias"], sel, z=c["z"], h_in=c["h_in"])
    for (b, h), o, hf in zip(sel, outs, hs):
        close(o, y[b, :, h])
        close(hf, hT[b, h])


# ---------------------------------------------------------------- conv + SiLU over x, B, C
def _np_conv_silu(x_bc, w_c, b_c, state_c=None):
    """One channel through numpy.convolve over the left-padded sequence, then SiLU."""
    K = w_c.shape[0]
    pad = np.zeros(K - 1) if state_c is None else np.asarray(state_c, dtype=np.float64)
    xpad = np.concatenate([pad, x_bc])
    pre = np.convolve(xpad, w_c[::-1], mode="valid") + b_c
    return silu(pre), xpad[-(K - 1):]


def test_conv_matches_numpy_convolve():
    r = np.random.default_rng(200)
    Bt, L, Cc, K = 2, 11, 5, 4
    x = r.standard_normal((Bt, L, Cc))
    w = r.standard_normal((Cc, K))
    bias = r.standard_normal(Cc)
    st = r.standard_normal((Bt, Cc, K - 1))
    out, cs = so.conv_silu(x, w, bias, conv_state_in=st)
    for b in range(Bt):
        for c in range(Cc):
            o, last = _np_conv_silu(x[b, :, c], w[c], bias[c], st[b, c])
            close(out[b, :, c], o)
            close(cs[b, c], last)
    out0, cs0 = so.conv_silu(x, w)
    o, last = _np_conv_silu(x[1, :, 3], w[3], 0.0)
    close(out0[1, :, 3], o)
    close(cs0[1, 3], last)


@pytest.mark.parametrize("L", [0, 1, 2, 3, 5])
def test_conv_state_out_orientation(L):
    r = np.random.default_rng(210 + L)
    x = r.standard_normal((1, L, 2))
    st = r.standard_normal((1, 2, 3))
    _, cs = so.conv_silu(x, r.standard_normal((2, 4)), conv_state_in=st)
    expect = np.concatenate([st[0].T, x[0]], axis=0)[-3:].T          # last 3 of [state; x]
    close(cs[0], expect)


def test_conv_packed_row_equals_documents():
    r = np.random.default_rng(220)
    L, Cc = 14, 3
    x = r.standard_normal((1, L, Cc))
    w = r.standard_normal((Cc, 4))
    bias = r.standard_normal(Cc)
    st = r.standard_normal((1, Cc, 3))
    ids = np.array([[4, 4, 4, 4, 4, 7, 7, 1, 1, 1, 1, 1, 1, 1]])
    out, cs = so.conv_silu(x, w, bias, seq_idx=ids, conv_state_in=st)
    o0, _ = so.conv_silu(x[:, 0:5], w, bias, conv_state_in=st)        # first document: the state
    o1, _ = so.conv_silu(x[:, 5:7], w, bias)
    o2, c2 = so.conv_silu(x[:, 7:], w, bias)
    close(out, np.concatenate([o0, o1, o2], axis=1))
    close(cs, c2)
    # a repeated id after another document still resets (changes count, not values)
    ids2 = np.array([[4, 4, 4, 4, 4, 7, 7, 4, 4, 4, 4, 4, 4, 4]])
    out2, _ = so.conv_silu(x, w, bias, seq_idx=ids2, conv_state_in=st)
    close(out2, out)
    # a short last document: the state slots before it are zero
    ids3 = np.array([[4] * 13 + [9]])
    _, cs3 = so.conv_silu(x, w, bias, seq_idx=ids3, conv_state_in=st)
    close(cs3[0, :, :2], np.zeros((Cc, 2)))
    close(cs3[0, :, 2], x[0, -1])


# ---------------------------------------------------------------- gated RMSNorm
def test_gated_rmsnorm_unit_mean_square_and_weight():
    r = np.random.default_rng(230)
    y, z = r.standard_normal((3, 5, 24)), r.standard_normal((3, 5, 24))
    out = so.gated_rmsnorm(y, z, np.ones(24), eps=0.0)
    close(np.mean(out ** 2, axis=-1), np.ones((3, 5)))                  # unit RMS per row
    g = y * expit(z) * z
    close(out * np.sqrt(np.mean(g ** 2, axis=-1, keepdims=True)), g)     # direction of the gated input
    w = r.standard_normal(24)
    close(so.gated_rmsnorm(y, z, w, eps=0.0), out * w)


def test_gated_rmsnorm_scale_invariance_and_eps():
    r = np.random.default_rng(240)
    y, z = r.standard_normal((4, 16)), r.standard_normal((4, 16))
    w = r.standard_normal(16)
    close(so.gated_rmsnorm(7.5 * y, z, w, eps=0.0), so.gated_rmsnorm(y, z, w, eps=0.0))
    # eps matters only against the mean square: a tiny input is pulled toward zero
    tiny = so.gated_rmsnorm(1e-4 * y, z, w, eps=1e-5)
    assert np.max(np.abs(tiny)) < 0.1 * np.max(np.abs(so.gated_rmsnorm(y, z, w, eps=1e-5)))


def test_gated_rmsnorm_groups_are_separate_norms():
    r = np.random.default_rng(250)
    y, z = r.standard_normal((2, 3, 32)), r.standard_normal((2, 3, 32))
    w = r.standard_normal(32)
    out = so.gated_rmsnorm(y, z, w, group_size=8)
    for gi in range(4):
        sl = slice(8 * gi, 8 * gi + 8)
        close(out[..., sl], so.gated_rmsnorm(y[..., sl], z[..., sl], w[sl]))


# ---------------------------------------------------------------- regression fixture
def test_oracle_matches_its_golden_fixture():
    """tests/golden/ssd_tiny_oracle_samples.json (written by tests/golden/make_golden_ssd.py
    from the oracle): a later change to the oracle's arithmetic shows up here (to 1e-12:
    numpy's exp and log may differ in the last bit between machines)."""
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(__file__), "golden")
    spec = importlib.util.spec_from_file_location("make_golden_ssd", os.path.join(here, "make_golden_ssd.py"))
    mk = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mk)
    g = json.load(open(os.path.join(here, "ssd_tiny_oracle_samples.json")))
    now = mk.compute()
    for key in ("y", "h_out", "conv", "norm"):
        for (ix, v), (ix2, v2) in zip(g[key], now[key]):
            assert ix == ix2
            assert abs(v - v2) <= 1e-12 * max(1.0, abs(v)), (key, ix, v, v2)
    np.testing.assert_allclose(now["conv_state_out_b0_c7"], g["conv_state_out_b0_c7"], rtol=1e-12, atol=0)


# ---------------------------------------------------------------- random shapes
def chunked_with_resets(c, Q, ids):
    """The chunked form with documents: within a chunk the mask also needs s and t in one
    document, the inter-chunk term of step t needs no reset in (chunk start, t], and the
    state update takes the chunk's last document only (zero carried decay after a reset)."""
    x, dtr, Bm, Cm = c["x"], c["dt_raw"], c["B"], c["C"]
    Bt, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    y = np.zeros((Bt, L, H, P))
    hT = np.zeros((Bt, H, P, N))
    for b in range(Bt):
        reset = np.zeros(L, dtype=bool)
        reset[1:] = ids[b, 1:] != ids[b, :-1]
        for h in range(H):
            g = h // (H // G)
            A = -np.exp(c["A_log"][h])
            Hs = np.zeros((P, N)) if c.get("h_in") is None else c["h_in"][b, h].copy()
            for c0 in range(0, L, Q):
                idx = np.arange(c0, min(L, c0 + Q))
                q = len(idx)
                last_reset = np.full(q, -1)
                lr = -1
                for i, t in enumerate(idx):
                    if reset[t]:
                        lr = i
                    last_reset[i] = lr
                dl = softplus(dtr[b, idx, h] + c["dt_bias"][h])
                cs = np.cumsum(dl * A)
                Mm = np.zeros((q, q))
                for i in range(q):
                    for j in range(max(last_reset[i], 0), i + 1):
                        Mm[i, j] = np.exp(cs[i] - cs[j]) * dl[j]
                inter = np.where(last_reset < 0, np.exp(cs), 0.0)
                Y = (Mm * (Cm[b, idx, g] @ Bm[b, idx, g].T)) @ x[b, idx, h] \
                    + inter[:, None] * (Cm[b, idx, g] @ Hs.T) + c["D"][h] * x[b, idx, h]
                if c.get("z") is not None:
                    Y = Y * silu(c["z"][b, idx, h])
                y[b, idx, h] = Y
                lo = max(last_reset[-1], 0)
                wl = np.where(np.arange(q) >= lo, np.exp(cs[-1] - cs) * dl, 0.0)
                dec = np.exp(cs[-1]) if last_reset[-1] < 0 else 0.0
                Hs = dec * Hs + (x[b, idx, h] * wl[:, None]).T @ Bm[b, idx, g]
            hT[b, h] = Hs
    return y, hT


from hypothesis import given, settings, strategies as st  # noqa: E402


@settings(max_examples=25, deadline=None)
@given(seed=st.integers(0, 10 ** 6), L=st.integers(1, 19), Q=st.integers(1, 8),
       G=st.sampled_from([1, 2]), hpg=st.integers(1, 2), P=st.integers(1, 3),
       N=st.integers(1, 4), gate=st.booleans(), state=st.booleans(), docs=st.integers(0, 4))
def test_random_shapes_chunked_and_unrolled(seed, L, Q, G, hpg, P, N, gate, state, docs):
    c = case(seed, Bt=2, L=L, H=G * hpg, P=P, N=N, G=G, z=gate, h_in=state)
    r = np.random.default_rng(seed + 1)
    ids = np.cumsum(r.random((2, L)) < docs / 10.0, axis=1)         # random document starts
    y, hT = run(c, seq_idx=ids)
    yc, hc = chunked_with_resets(c, Q, ids)
    close(y, yc, 1e-10)
    close(hT, hc, 1e-10)
    yu, hu = unrolled(c, seq_idx=ids)
    close(y, yu, 1e-10)
    close(hT, hu, 1e-10)
