"""GPU parity of the backward (mamba_mixer_bwd through the C ABI) with the fp64 backward
oracle (pinned against finite differences in test_oracle_bwd.py): every gradient, element
by element, in the gradient tolerance of tests/tolerances.py, on several tiles with
ragged channel and time tails, in fp32 and bf16, d_state 16 and 8, with and without a conv
bias; the 130M-class shape on sampled channels."""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import host, to_device
from tests.gpu_util import oracle_full
from tests.tolerances import assert_close, assert_close_grad

pytestmark = pytest.mark.gpu


def _case(Bt, L, Di, N, io, seed, conv_b=True):
    w = I.Workload("bwd", Bt, L, Di, N, 4, io, seed)
    inp = I.make_inputs(w)
    if not conv_b:
        inp["conv_b"] = None
    r = np.random.default_rng(seed + 1)
    dy = r.standard_normal((Bt, L, Di)).astype(np.float32)
    inp["dy"] = I.f32_to_bf16_bits(dy) if io == I.BF16 else dy
    return w, inp


def _run(inp):
    d = to_device(inp)
    g = M.mamba_mixer_bwd(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                          d["conv_w"], d.get("conv_b"), d["dt_bias"], d["dy"])
    torch.cuda.synchronize()
    return {k: (None if v is None else host(v)) for k, v in g.items()}


def _oracle(oracle, inp):
    w = I.as_f64
    return oracle.mixer_bwd(w(inp["xp"]), w(inp["z"]), w(inp["dt_raw"]), w(inp["B"]),
                            w(inp["C"]), inp["A_log"], inp["D"], inp["conv_w"], inp.get("conv_b"),
                            inp["dt_bias"], w(inp["dy"]), nthreads=0)


def _compare(g, go, io, what):
    for k in M.BWD_OUTPUTS:
        if go[k] is None:
            assert g[k] is None
            continue
        assert_close_grad(g[k], go[k], io, f"{what} {k}")


@pytest.mark.parametrize("Bt,L,Di,N,io,conv_b", [
    (2, 16, 128, 16, I.F32, True),      # tiny config shape
    (2, 77, 72, 16, I.F32, False),      # ragged time and channel tails
    (3, 300, 64, 16, I.BF16, True),
    (2, 129, 104, 8, I.BF16, True),
    (2, 64, 40, 8, I.F32, True),
])
def test_backward_matches_oracle(oracle, Bt, L, Di, N, io, conv_b):
    w, inp = _case(Bt, L, Di, N, io, 3000 + L + Di, conv_b)
    _compare(_run(inp), _oracle(oracle, inp), io, f"{Bt}x{L}x{Di} N{N} {io}")


def test_backward_130m_two_rows(oracle):
    """Two batch rows of the 130M-class layer (2 x 2048 x 1536, bf16): every gradient in
    full, including dB/dC (sums over all 1536 channels) and the parameter gradients."""
    w, inp = _case(2, 2048, 1536, 16, I.BF16, 3100)
    _compare(_run(inp), _oracle(oracle, inp), I.BF16, "m130 rows")


@pytest.mark.parametrize("Bt,L,Di,N,io", [
    (1, 4096, 64, 16, I.BF16),     # 16 chunks of 256 steps
    (2, 1500, 64, 8, I.F32),       # 5 chunks of 320 steps, the last one ragged
    (1, 2600, 40, 16, I.F32),      # ragged channel tile and sequence
])
def test_backward_with_time_chunks(oracle, Bt, L, Di, N, io):
    """Rows with few channel tiles are cut into time chunks: the state and the adjoint are
    carried across chunk edges, and the input gradient of each chunk's last 3 steps takes
    the next chunk's part."""
    dims = M.make_dims(Bt, L, Di, N, 4, M.MAMBA_BF16 if io == I.BF16 else M.MAMBA_F32)
    # the backward's plan splits the sequence: its workspace holds per-chunk aggregates
    # beyond the header and the per-tile start states
    per = Bt * Di * N * 4
    assert M.mamba_mixer_bwd_workspace_bytes(dims) > 256 + (L + 15) // 16 * per
    w, inp = _case(Bt, L, Di, N, io, 3200 + L)
    _compare(_run(inp), _oracle(oracle, inp), io, f"chunked {Bt}x{L}x{Di} N{N} {io}")


def test_backward_long_sampled_channels(oracle):
    """The long-sequence shape in full (2 x 65536 x 2560, bf16; 12 time chunks): every
    gradient of a channel depends only on that channel and B/C, so the per-channel
    gradients (dxp, dz, ddt_raw and the parameter gradients) of sampled channels are checked
    against the oracle run on those channels alone; dB/dC (sums over all channels) are
    covered by the other tests."""
    from tests.gpu_util import pick_channels
    w, inp = _case(2, 65536, 2560, 16, I.BF16, 3300)
    di = pick_channels(2560, 10, 5)
    d = to_device(inp)
    gd = M.mamba_mixer_bwd(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                           d["conv_w"], d["conv_b"], d["dt_bias"], d["dy"])
    torch.cuda.synchronize()
    idx = torch.as_tensor(di, device="cuda")
    g = {k: host(v[:, :, idx] if v.dim() == 3 and k in ("dxp", "dz", "ddt_raw") else v)
         for k, v in gd.items() if k not in ("dB", "dC")}
    del gd, d
    sub = dict(inp)
    for k in ("xp", "z", "dt_raw", "dy"):
        sub[k] = inp[k][:, :, di]
    for k in ("A_log", "D", "conv_w", "conv_b", "dt_bias"):
        sub[k] = inp[k][di]
    go = _oracle(oracle, sub)
    for k in ("dxp", "dz", "ddt_raw"):
        assert_close_grad(g[k], go[k], I.BF16, f"long {k}")
    for k in ("dA_log", "dD", "dconv_w", "dconv_b", "ddt_bias"):
        assert_close_grad(g[k][di], go[k], I.BF16, f"long {k}")


def _case_packed(Bt, L, Di, N, io, seed, case, state, edge):
    w = I.Workload("bwdp", Bt, L, Di, N, 4, io, seed, decode=state)
    inp = I.make_inputs(w)
    dy = np.random.default_rng(seed + 1).standard_normal((Bt, L, Di)).astype(np.float32)
    inp["dy"] = I.f32_to_bf16_bits(dy) if io == I.BF16 else dy
    inp["seq_idx"] = None if case is None else I.seq_idx_case(case, Bt, L, edge=edge, seed=9)
    return w, inp


def _run_packed(inp, state):
    d = to_device({k: v for k, v in inp.items() if k != "seq_idx"})
    seq = None if inp["seq_idx"] is None else torch.from_numpy(inp["seq_idx"]).cuda()
    g = M.mamba_mixer_bwd_packed(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                                 d["conv_w"], d.get("conv_b"), d["dt_bias"], d["dy"], seq_idx=seq,
                                 h_in=d["h"] if state else None,
                                 conv_state_in=d["conv_state"] if state else None)
    torch.cuda.synchronize()
    return {k: (None if v is None else host(v)) for k, v in g.items()}


def _oracle_packed(oracle, inp, state):
    w = I.as_f64
    return oracle.mixer_bwd(w(inp["xp"]), w(inp["z"]), w(inp["dt_raw"]), w(inp["B"]), w(inp["C"]),
                            inp["A_log"], inp["D"], inp["conv_w"], inp.get("conv_b"),
                            inp["dt_bias"], w(inp["dy"]), nthreads=0, seq_idx=inp["seq_idx"],
                            h_in=inp["h"] if state else None,
                            conv_state_in=w(inp["conv_state"]) if state else None)


def _compare_packed(g, go, io, what):
    _compare(g, go, io, what)
    for k in ("dh_in", "dconv_state_in"):
        if go[k] is None:
            # no cached start in the forward: the device still returns the zero-input gradient
            continue
        assert_close_grad(g[k], go[k], io, f"{what} {k}")


@pytest.mark.parametrize("state", [False, True])
@pytest.mark.parametrize("io", [I.F32, I.BF16])
@pytest.mark.parametrize("case", ["length_one_docs", "consecutive_boundaries", "boundary_on_edge",
                                  "terminal_padding", "many_short_docs"])
def test_packed_backward_matches_oracle(oracle, case, io, state):
    w, inp = _case_packed(3, 300, 64, 16, io, 3400 + len(case), case, state, edge=16)
    _compare_packed(_run_packed(inp, state), _oracle_packed(oracle, inp, state), io,
                    f"packed {case} {io} state={state}")


@pytest.mark.parametrize("case", ["boundary_on_edge", "many_short_docs", "misaligned_rows"])
def test_packed_backward_with_time_chunks(oracle, case):
    """16 chunks of 256 steps with boundaries on the chunk edges (and everywhere)."""
    w, inp = _case_packed(2, 4096, 64, 16, I.BF16, 3500 + len(case), case, True, edge=256)
    dims = M.make_dims(2, 4096, 64, 16, 4, M.MAMBA_BF16)    # the backward's plan chunks it
    assert M.mamba_mixer_bwd_workspace_bytes(dims) > 256 + 4096 // 16 * 2 * 64 * 16 * 4
    _compare_packed(_run_packed(inp, True), _oracle_packed(oracle, inp, True), I.BF16,
                    f"packed chunked {case}")


def test_packed_backward_cached_start_only(oracle):
    """No documents, a cached start: the state gradients against the oracle's."""
    w, inp = _case_packed(2, 777, 72, 8, I.F32, 3600, None, True, edge=16)
    _compare_packed(_run_packed(inp, True), _oracle_packed(oracle, inp, True), I.F32, "cached")


@pytest.mark.parametrize("io", [I.F32, I.BF16])
def test_autograd_function_matches_oracle(oracle, io):
    """mixer.mamba_mixer as a torch autograd op: y.backward(dy) fills every input's .grad
    (in the input's dtype) with the oracle's gradients."""
    w, inp = _case(2, 200, 64, 16, io, 3700)
    d = to_device(inp)
    names = ("xp", "z", "dt_raw", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias")
    leaves = {k: d[k].clone().requires_grad_(True) for k in names}
    y = M.mamba_mixer(*(leaves[k] for k in names))
    y.backward(d["dy"])
    torch.cuda.synchronize()
    go = _oracle(oracle, inp)
    for k in names:
        assert leaves[k].grad is not None and leaves[k].grad.dtype == leaves[k].dtype, k
        # bf16 gradients of activations carry bf16 rounding on top of the fp32 result
        assert_close_grad(host(leaves[k].grad), go["d" + k], io,
                          f"autograd {io} {k}")


# ---- the training pair with state checkpoints (mamba_mixer_fwd_ckpt / mamba_mixer_bwd_ckpt)

@pytest.mark.parametrize("Bt,L,Di,N,io", [
    (12, 200, 1024, 16, I.BF16),   # 384 channel tiles: the prep/scan forward kernel
    (2, 4100, 96, 16, I.BF16),     # few tiles: four time groups, chained chunks, ragged tail
    (3, 300, 64, 8, I.BF16),       # four time groups, one chunk, d_state 8
    (2, 77, 72, 16, I.F32),        # fp32, ragged time and channel tails
    (1, 2600, 40, 16, I.F32),      # fp32 with a chunk-state pass (time chunks)
])
def test_checkpointed_backward_matches_oracle(oracle, Bt, L, Di, N, io):
    """The forward that writes the state before every 16-step tile gives the same y as the
    plain forward (bit for bit), its checkpoints start from zero and match the oracle's
    state after each 16-step prefix, and the backward that reads them matches the oracle
    in the gradient tolerance."""
    w, inp = _case(Bt, L, Di, N, io, 3400 + L + Di)
    d = to_device(inp)
    args = (d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"], d["conv_w"],
            d.get("conv_b"), d["dt_bias"])
    dims = M.make_dims(Bt, L, Di, N, 4, M.MAMBA_BF16 if io == I.BF16 else M.MAMBA_F32)
    ck = M.new_ckpt(dims, d["xp"].device)
    assert ck.numel() * 4 == M.load_library().mamba_mixer_ckpt_bytes(__import__("ctypes").byref(dims))
    ck.fill_(float("nan"))                   # every entry must be written
    y_ck, h_ck, _ = M.mamba_mixer_fwd(*args, h_ckpt=ck)
    y, h, _ = M.mamba_mixer_fwd(*args)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(host(y_ck), host(y))
    np.testing.assert_array_equal(host(h_ck), host(h))
    ckh = host(ck)
    assert np.isfinite(ckh).all()
    assert (ckh[:, 0] == 0).all()
    # the oracle's state after 16k steps, for a few k (prefix runs)
    rng = np.random.default_rng(L)
    t16 = (L + 15) // 16
    for k in sorted(set([1, t16 - 1] + [int(v) for v in rng.integers(1, t16, 2)])):
        if k < 1 or k >= t16:
            continue
        pre = {key: (np.ascontiguousarray(v[:, :16 * k]) if key in ("xp", "z", "dt_raw", "B", "C")
                     else v) for key, v in inp.items() if key != "dy"}
        _, ho, _ = oracle_full(oracle, pre)
        assert_close(ckh[:, k], ho, io, f"checkpoint {k} (state after {16 * k} steps)")
    g = M.mamba_mixer_bwd(*args, d["dy"], h_ckpt=ck)
    torch.cuda.synchronize()
    g = {k: (None if v is None else host(v)) for k, v in g.items()}
    _compare(g, _oracle(oracle, inp), io, f"checkpointed {Bt}x{L}x{Di} N{N} {io}")


def test_checkpointed_autograd_matches_recompute(oracle):
    """MambaMixerFunction with checkpoint_states gives the recomputing path's gradients in
    the gradient tolerance of each other and of the oracle."""
    w, inp = _case(2, 300, 256, 16, I.BF16, 3500)
    d = to_device(inp)
    outs = []
    for ckpt in (False, True):
        leaves = {k: d[k].clone().requires_grad_(d[k].dtype.is_floating_point)
                  for k in ("xp", "z", "dt_raw", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias")}
        y = M.mamba_mixer(*(leaves[k] for k in ("xp", "z", "dt_raw", "B", "C", "A_log", "D",
                                                "conv_w", "conv_b", "dt_bias")),
                          checkpoint_states=ckpt)
        y.backward(d["dy"])
        outs.append({k: host(v.grad.float()) for k, v in leaves.items()})
    go = _oracle(oracle, inp)
    names = {"xp": "dxp", "z": "dz", "dt_raw": "ddt_raw", "B": "dB", "C": "dC", "A_log": "dA_log",
             "D": "dD", "conv_w": "dconv_w", "conv_b": "dconv_b", "dt_bias": "ddt_bias"}
    for k, gk in names.items():
        assert_close_grad(outs[1][k], go[gk], I.BF16, f"checkpointed autograd {k}")
        assert_close_grad(outs[1][k], outs[0][k], I.BF16, f"checkpointed vs recompute {k}")
