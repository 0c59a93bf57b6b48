"""Parity of the Mamba2 scan (mamba2_ssd_fwd, CUDA, through the C ABI) with the fp64 oracle.

Shapes span several 64-step chunks with ragged tails, both supported d_state values, one
and several groups, the gate, an initial state (also updated in place), the empty and
single-step sequences, rows packing documents (the nine structural seq_idx cases of
niverel-mamba 0.1.0, section "seq_idx strict reset", with and without an initial state and
time segments), and the reference layer (24 heads x 64, d_state 128) at full size on
sampled (batch row, head) pairs.  Tolerance: tests/tolerances.py assert_close_tc.
"""

import numpy as np
import pytest
import torch

from oracle import ssd_oracle as so
from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import ssd as S
from tests.gpu_util import dev_tensor, host
from tests.tolerances import assert_close_tc

pytestmark = pytest.mark.gpu


def draw(Bt, L, H, N, G, gate, state, seed):
    w = I.SsdWorkload("case", Bt, L, H, 64, N, G, seed, gate=gate, state=state)
    return I.make_ssd_inputs(w)


def run_gpu(inp, h_in_inplace=False, seq_idx=None):
    d = {k: (None if v is None else dev_tensor(v)) for k, v in inp.items()}
    h_out = d["h_in"] if h_in_inplace else None
    ids = None if seq_idx is None else torch.from_numpy(np.ascontiguousarray(seq_idx, dtype=np.int32)).cuda()
    y, h = S.mamba2_ssd_fwd(d["x"], d["dt_raw"], d["A_log"], d["B"], d["C"], d["D"],
                            d["dt_bias"], z=d["z"], seq_idx=ids, h_in=d["h_in"], h_out=h_out)
    torch.cuda.synchronize()
    return host(y), host(h)


def run_oracle(inp, seq_idx=None):
    return so.ssd(inp["x"], inp["dt_raw"], inp["A_log"], inp["B"], inp["C"], inp["D"],
                  inp["dt_bias"], z=inp["z"], h_in=inp["h_in"], seq_idx=seq_idx)


CASES = [
    # Bt, L, H, N, G, gate, state
    (2, 100, 4, 64, 1, True, False),
    (1, 257, 3, 128, 1, False, True),
    (2, 64, 4, 128, 2, True, True),
    (1, 63, 2, 128, 1, False, False),
    (3, 130, 6, 64, 3, True, False),
    (1, 1, 2, 64, 1, True, True),
    (2, 200, 8, 128, 4, False, False),
    (1, 640, 2, 128, 1, True, True),
    # time segments (state pass) at d_state 64 with a carried-in state
    (1, 300, 2, 64, 1, False, True),
    # segments over a ragged last chunk (1100 = 17 x 64 + 12), gated, carried-in state
    (2, 1100, 3, 128, 1, True, True),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: "x".join(map(str, c)))
def test_ssd_matches_oracle(case):
    Bt, L, H, N, G, gate, state = case
    inp = draw(Bt, L, H, N, G, gate, state, seed=3000 + sum(case[:5]))
    y, h = run_gpu(inp)
    yo, ho = run_oracle(inp)
    assert_close_tc(y, yo, "y")
    assert_close_tc(h, ho, "h_out")


def test_state_in_place():
    inp = draw(2, 150, 4, 128, 1, False, True, seed=3100)
    yo, ho = run_oracle(inp)
    y, h = run_gpu(inp, h_in_inplace=True)
    assert_close_tc(y, yo, "y")
    assert_close_tc(h, ho, "h_out in place")


def test_status_word_is_clear_after_clean_calls():
    """The tensor-core pass (rows without document ids) waits on its own copies and products
    with bounded waits; after clean calls (one segment and several) mamba2_ssd_check finds
    no timeout, and calls with document ids (the other pass) leave it clear as well."""
    S.mamba2_ssd_check()                                  # start from a clear word
    for L in (300, 4096):
        run_gpu(draw(1, L, 2, 128, 1, True, True, seed=3150 + L))
    ids = np.zeros((2, 130), dtype=np.int32)
    ids[:, 70:] = 1                                       # one document change per row
    run_gpu(draw(2, 130, 4, 64, 1, False, False, seed=3151), seq_idx=ids)
    torch.cuda.synchronize()
    S.mamba2_ssd_check()


def test_empty_sequence_passes_state_through():
    inp = draw(2, 0, 4, 64, 1, True, True, seed=3200)
    y, h = run_gpu(inp)
    assert y.size == 0
    assert np.array_equal(h, inp["h_in"].astype(np.float64))
    inp["h_in"] = None
    _, h = run_gpu(inp)
    assert np.array_equal(h, np.zeros_like(h))


def test_prefix_then_continue():
    # a sequence split at a non-chunk boundary: the second call starts from the first's state
    inp = draw(1, 300, 4, 128, 1, True, False, seed=3300)
    yo, ho = run_oracle(inp)
    cut = 137
    first = {k: (v[:, :cut] if k in ("x", "dt_raw", "B", "C", "z") else v) for k, v in inp.items()}
    y1, h1 = run_gpu(first)
    second = {k: (np.ascontiguousarray(v[:, cut:]) if k in ("x", "dt_raw", "B", "C", "z") else v)
              for k, v in inp.items()}
    second["h_in"] = h1.astype(np.float32)
    y2, h2 = run_gpu(second)
    assert_close_tc(np.concatenate([y1, y2], axis=1), yo, "y (two calls)")
    assert_close_tc(h2, ho, "h_out (two calls)")


@pytest.mark.parametrize("name", ["ssd_v3", "ssd_v3_long"])
def test_reference_layer_full_size_sampled(name):
    w = I.SSD_WORKLOADS[name]
    inp = I.make_ssd_inputs(w)
    y, h = run_gpu(inp)
    assert np.isfinite(y).all() and np.isfinite(h).all()
    rng = np.random.default_rng(7)
    sel = [(int(rng.integers(w.batch)), int(rng.integers(w.nheads))) for _ in range(4)]
    sel += [(0, 0), (w.batch - 1, w.nheads - 1)]
    outs, hs = so.ssd_channels(inp["x"], inp["dt_raw"], inp["A_log"], inp["B"], inp["C"],
                               inp["D"], inp["dt_bias"], sel, z=inp["z"], h_in=inp["h_in"])
    for (b, hh), o, hf in zip(sel, outs, hs):
        assert_close_tc(y[b, :, hh], o, f"y[{b}, :, {hh}]")
        assert_close_tc(h[b, hh], hf, f"h_out[{b}, {hh}]")


@pytest.mark.parametrize("name", I.SEQ_IDX_CASES)
@pytest.mark.parametrize("state", [False, True])
def test_packed_documents(name, state):
    Bt, L, H = 2, 200, 4
    inp = draw(Bt, L, H, 128, 1, True, state, seed=3400 + I.SEQ_IDX_CASES.index(name))
    ids = I.seq_idx_case(name, Bt, L, edge=64, seed=9)
    yo, ho = run_oracle(inp, ids)
    y, h = run_gpu(inp, seq_idx=ids)
    assert_close_tc(y, yo, f"y ({name})")
    assert_close_tc(h, ho, f"h_out ({name})")


def test_packed_long_row_sampled():
    # 2 rows of 8192 steps packing documents of mean length 256, time segments on
    w = I.SsdWorkload("packed_long", 2, 8192, 24, 64, 128, 1, 3500, state=True)
    inp = I.make_ssd_inputs(w)
    ids = I.packed_seq_idx(2, 8192, 256, 3501)
    y, h = run_gpu(inp, seq_idx=ids)
    sel = [(0, 0), (1, 23), (0, 11), (1, 5)]
    outs, hs = so.ssd_channels(inp["x"], inp["dt_raw"], inp["A_log"], inp["B"], inp["C"],
                               inp["D"], inp["dt_bias"], sel, z=inp["z"], h_in=inp["h_in"],
                               seq_idx=ids)
    for (b, hh), o, hf in zip(sel, outs, hs):
        assert_close_tc(y[b, :, hh], o, f"y[{b}, :, {hh}]")
        assert_close_tc(h[b, hh], hf, f"h_out[{b}, {hh}]")


PACKED_VARIANTS = [
    # name, Bt, L, H, N, G, gate, state, in_place
    ("many_short_docs", 3, 300, 4, 64, 2, True, True, False),
    ("misaligned_rows", 1, 700, 2, 64, 1, False, True, True),
    ("consecutive_boundaries", 2, 130, 6, 128, 3, True, False, False),
    ("terminal_padding", 2, 513, 2, 128, 2, True, True, True),
]


@pytest.mark.parametrize("case", PACKED_VARIANTS, ids=lambda c: c[0] + "-" + "x".join(map(str, c[1:])))
def test_packed_variants(case):
    name, Bt, L, H, N, G, gate, state, in_place = case
    inp = draw(Bt, L, H, N, G, gate, state, seed=3600 + L)
    ids = I.seq_idx_case(name, Bt, L, edge=64, seed=11)
    yo, ho = run_oracle(inp, ids)
    y, h = run_gpu(inp, h_in_inplace=in_place, seq_idx=ids)
    assert_close_tc(y, yo, f"y ({name})")
    assert_close_tc(h, ho, f"h_out ({name})")


# ---------------------------------------------------------------- decode step
def run_step(inp, in_place=False):
    d = {k: (None if v is None else dev_tensor(v)) for k, v in inp.items()}
    h_out = d["h_in"] if in_place else None
    y, h = S.mamba2_ssd_step(d["x"], d["dt_raw"], d["A_log"], d["B"], d["C"], d["D"],
                             d["dt_bias"], d["h_in"], z=d["z"], h_out=h_out)
    torch.cuda.synchronize()
    return host(y), host(h)


@pytest.mark.parametrize("case", [(3, 4, 128, 1, True, False), (5, 6, 64, 3, False, True),
                                  (1, 1, 64, 1, True, True), (2, 8, 128, 4, False, False)],
                         ids=lambda c: "x".join(map(str, c)))
def test_step_matches_oracle(case):
    Bt, H, N, G, gate, in_place = case
    inp = draw(Bt, 1, H, N, G, gate, True, seed=3700 + Bt * H)
    yo, ho = run_oracle(inp)
    y, h = run_step(inp, in_place)
    assert_close_tc(y, yo, "step y")
    assert_close_tc(h, ho, "step h")


def test_prefill_then_steps_equal_forward():
    # niverel-mamba 0.1.0, "Autoregressive decoding": concatenated steps equal the forward
    Bt, L, H, N, k = 2, 100, 4, 128, 7
    inp = draw(Bt, L, H, N, 2, True, True, seed=3800)
    yo, ho = run_oracle(inp)
    acts = ("x", "dt_raw", "B", "C", "z")
    pre = {kk: (np.ascontiguousarray(v[:, :L - k]) if kk in acts else v) for kk, v in inp.items()}
    y1, h = run_gpu(pre)
    ys = [y1]
    for t in range(L - k, L):
        one = {kk: (np.ascontiguousarray(v[:, t:t + 1]) if kk in acts else v) for kk, v in inp.items()}
        one["h_in"] = h.astype(np.float32)
        yt, h = run_step(one, in_place=True)
        ys.append(yt)
    assert_close_tc(np.concatenate(ys, axis=1), yo, "prefill + steps y")
    assert_close_tc(h, ho, "prefill + steps h")


# ---------------------------------------------------------------- the layer around the scan
from tests.tolerances import assert_close  # noqa: E402


def draw_layer(Bt, L, H, N, G, seed, state=True):
    r = np.random.default_rng(seed)
    Cc = H * 64 + 2 * G * N
    return dict(
        xbc=I.f32_to_bf16_bits(r.standard_normal((Bt, L, Cc)).astype(np.float32)),
        conv_w=r.uniform(-0.5, 0.5, size=(Cc, 4)).astype(np.float32),
        conv_b=r.uniform(-0.5, 0.5, size=Cc).astype(np.float32),
        cs_in=I.f32_to_bf16_bits(r.standard_normal((Bt, Cc, 3)).astype(np.float32)) if state else None,
    )


@pytest.mark.parametrize("case", [(2, 150, 4, 64, 1, None, True), (1, 2, 2, 128, 2, "length_one_docs", True),
                                  (2, 200, 6, 128, 3, "many_short_docs", False),
                                  (1, 130, 2, 64, 1, "boundary_on_edge", True), (2, 0, 2, 64, 1, None, True)],
                         ids=lambda c: "x".join(map(str, c)))
def test_conv_silu_matches_oracle(case):
    Bt, L, H, N, G, name, state = case
    inp = draw_layer(Bt, L, H, N, G, seed=3900 + L + H, state=state)
    ids = None if name is None else I.seq_idx_case(name, Bt, L, edge=64, seed=5)
    ref, cs_ref = so.conv_silu(inp["xbc"], inp["conv_w"], inp["conv_b"], seq_idx=ids,
                               conv_state_in=inp["cs_in"])
    d = {k: (None if v is None else dev_tensor(v)) for k, v in inp.items()}
    tid = None if ids is None else torch.from_numpy(ids.astype(np.int32)).cuda()
    x, B, C, cs = S.mamba2_conv_silu(d["xbc"], d["conv_w"], d["conv_b"], nheads=H, ngroups=G,
                                     d_state=N, seq_idx=tid, conv_state_in=d["cs_in"])
    torch.cuda.synchronize()
    got = np.concatenate([host(x).reshape(Bt, L, H * 64), host(B).reshape(Bt, L, G * N),
                          host(C).reshape(Bt, L, G * N)], axis=2)
    assert_close(got, ref, "bf16", "conv + SiLU")
    np.testing.assert_array_equal(host(cs), cs_ref)   # a copy of inputs (or zeros): bitwise


@pytest.mark.parametrize("case", [(2, 50, 24, 1), (3, 17, 8, 2), (1, 5, 6, 3)],
                         ids=lambda c: "x".join(map(str, c)))
def test_gated_rmsnorm_matches_oracle(case):
    Bt, L, H, G = case
    r = np.random.default_rng(4000 + H)
    y = I.f32_to_bf16_bits(r.standard_normal((Bt, L, H * 64)).astype(np.float32))
    z = I.f32_to_bf16_bits(r.standard_normal((Bt, L, H * 64)).astype(np.float32))
    w = r.standard_normal(H * 64).astype(np.float32)
    ref = so.gated_rmsnorm(y, z, w, 1e-5, group_size=H * 64 // G)
    out = S.mamba2_gated_rmsnorm(dev_tensor(y), dev_tensor(z), dev_tensor(w), 1e-5, ngroups=G)
    torch.cuda.synchronize()
    assert_close(host(out), ref, "bf16", "gated RMSNorm")


def test_layer_conv_scan_norm_matches_oracle():
    # everything between the projections: conv + SiLU over x|B|C, the scan with a gate-free
    # output, then the gated RMSNorm (the rmsnorm=True layer of the weight contract)
    Bt, L, H, N, G = 2, 300, 4, 128, 1
    lay = draw_layer(Bt, L, H, N, G, seed=4100)
    w = I.SsdWorkload("layer", Bt, L, H, 64, N, G, 4101, gate=True)
    scan = I.make_ssd_inputs(w)
    ids = I.packed_seq_idx(Bt, L, 80, 4102)
    nw = np.random.default_rng(4103).standard_normal(H * 64).astype(np.float32)
    # oracle chain (the oracle's conv output rounded to bf16, as the scan takes it)
    conv_ref, _ = so.conv_silu(lay["xbc"], lay["conv_w"], lay["conv_b"], seq_idx=ids,
                               conv_state_in=lay["cs_in"])
    cb = I.f32_to_bf16_bits(conv_ref.astype(np.float32))
    xr = cb[..., :H * 64].reshape(Bt, L, H, 64)
    Br = np.ascontiguousarray(cb[..., H * 64:H * 64 + G * N]).reshape(Bt, L, G, N)
    Cr = np.ascontiguousarray(cb[..., H * 64 + G * N:]).reshape(Bt, L, G, N)
    yr, _ = so.ssd(xr, scan["dt_raw"], scan["A_log"], Br, Cr, scan["D"], scan["dt_bias"],
                   seq_idx=ids)
    yb = I.f32_to_bf16_bits(yr.astype(np.float32))
    ref = so.gated_rmsnorm(yb.reshape(Bt, L, -1), scan["z"].reshape(Bt, L, -1), nw, 1e-5)
    # the library
    d = {k: (None if v is None else dev_tensor(v)) for k, v in lay.items()}
    tid = torch.from_numpy(ids.astype(np.int32)).cuda()
    x, B, C, _ = S.mamba2_conv_silu(d["xbc"], d["conv_w"], d["conv_b"], nheads=H, ngroups=G,
                                    d_state=N, seq_idx=tid, conv_state_in=d["cs_in"])
    sd = {k: (None if v is None else dev_tensor(v)) for k, v in scan.items()}
    y, _ = S.mamba2_ssd_fwd(x, sd["dt_raw"], sd["A_log"], B, C, sd["D"], sd["dt_bias"], seq_idx=tid)
    out = S.mamba2_gated_rmsnorm(y, sd["z"], dev_tensor(nw), 1e-5)
    torch.cuda.synchronize()
    assert_close_tc(host(out).reshape(Bt, L, H * 64), ref, "layer output")
