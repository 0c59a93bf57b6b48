"""GPU parity of the fused forward (mamba_mixer_fwd through the C ABI) with the oracle.

Element-by-element on the five workloads' forward shapes (in full where the oracle is
quick, on sampled channels -- every time step of each sampled channel -- at full size),
plus ragged and degenerate shapes, random parameters, the kill-selectivity control,
determinism, non-finite propagation and guard bands around every output.
"""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from tests.gpu_util import (gpu_fwd, host, host_bits, oracle_full,
                            pick_channels, to_device)
from tests.tolerances import assert_close, same_nonfinite_pattern

pytestmark = pytest.mark.gpu


def _check_full(oracle, w: I.Workload, inp=None, what=""):
    inp = inp if inp is not None else I.make_inputs(w)
    d = to_device(inp)
    y, h, cs = gpu_fwd(d)
    torch.cuda.synchronize()
    yo, ho, cso = oracle_full(oracle, inp)
    r = assert_close(host(y), yo, w.io_dtype, f"{what or w.name} y")
    assert_close(host(h), ho, w.io_dtype, f"{what or w.name} h_out")
    np.testing.assert_array_equal(host(cs), cso)   # conv state is a copy: bitwise
    return r


def _check_sampled(oracle, w: I.Workload, nb, nch, seed, inp=None):
    inp = inp if inp is not None else I.make_inputs(w)
    d = to_device(inp)
    y, h, cs = gpu_fwd(d)
    torch.cuda.synchronize()
    bi = np.unique(np.r_[0, w.batch - 1, np.random.default_rng(seed).integers(0, w.batch, nb)])
    di = pick_channels(w.d_inner, nch, seed)
    yo, ho, cso = oracle.mixer_channels(inp, bi, di, widen=I.as_f64, nthreads=0)
    yg = host(y[torch.as_tensor(bi, device="cuda")][:, :, torch.as_tensor(di, device="cuda")])
    hg = host(h)[bi][:, di]
    csg = host(cs)[bi][:, di]
    r = assert_close(yg, yo, w.io_dtype, f"{w.name} y (sampled)")
    assert_close(hg, ho, w.io_dtype, f"{w.name} h_out (sampled)")
    np.testing.assert_array_equal(csg, cso)
    return r


def test_tiny_fp32(oracle):
    _check_full(oracle, I.WORKLOADS["tiny"])


def test_stress_fp32(oracle):
    _check_full(oracle, I.WORKLOADS["stress"])


def test_m130_bf16_sampled(oracle):
    _check_sampled(oracle, I.WORKLOADS["m130"], nb=8, nch=96, seed=1)


def test_long_bf16_sampled(oracle):
    """L = 65536: exercises the carry between time chunks on every sampled channel."""
    _check_sampled(oracle, I.WORKLOADS["long"], nb=2, nch=24, seed=2)


@pytest.mark.slow
def test_m130_bf16_full(oracle):
    _check_full(oracle, I.WORKLOADS["m130"])


@pytest.mark.parametrize("L", [0, 1, 2, 3, 4, 5, 17, 63, 64, 65, 1023, 1024, 1500, 3000, 4097])
def test_ragged_lengths_bf16(oracle, L):
    w = I.WORKLOADS["m130"].with_(batch=3, seqlen=L, d_inner=64, seed=50 + L)
    _check_full(oracle, w, what=f"L={L}")


@pytest.mark.parametrize("L", [0, 1, 3, 17, 2500])
def test_ragged_lengths_fp32(oracle, L):
    w = I.WORKLOADS["tiny"].with_(batch=2, seqlen=L, d_inner=40, seed=80 + L)
    _check_full(oracle, w, what=f"fp32 L={L}")


@pytest.mark.parametrize("Di", [8, 24, 136, 264])
def test_ragged_channels(oracle, Di):
    w = I.WORKLOADS["m130"].with_(batch=2, seqlen=300, d_inner=Di, seed=90 + Di)
    _check_full(oracle, w, what=f"Di={Di}")


@pytest.mark.parametrize("io,N", [("bf16", 8), ("f32", 16), ("f32", 8), ("bf16", 16)])
def test_state_sizes_and_dtypes(oracle, io, N):
    w = I.Workload("case", 2, 777, 96, N, 4, io, 123)
    _check_full(oracle, w, what=f"{io} N={N}")


def test_random_parameters_and_no_conv_bias(oracle):
    w = I.WORKLOADS["m130"].with_(batch=2, seqlen=1200, d_inner=128, seed=7)
    inp = I.make_inputs(w)
    inp.update(I.random_params(w, 8))
    inp["conv_b"] = None
    _check_full(oracle, w, inp, "random A_log/D, no conv bias")
    wf = I.WORKLOADS["stress"]
    inpf = I.make_inputs(wf)
    inpf.update(I.random_params(wf, 9))
    _check_full(oracle, wf, inpf, "stress random A_log/D")


def test_kill_selectivity_control(oracle):
    """Time-constant dt/B/C (the values at t = 0) must change the outputs far beyond the
    tolerance, and the GPU must still match the oracle on the killed inputs."""
    w = I.WORKLOADS["m130"].with_(batch=2, seqlen=256, d_inner=256, seed=11)
    inp = I.make_inputs(w)
    killed = dict(inp)
    for k in ("dt_raw", "B", "C"):
        killed[k] = np.ascontiguousarray(np.repeat(inp[k][:, :1], w.seqlen, axis=1))
    y_sel = host(gpu_fwd(to_device(inp))[0])
    _check_full(oracle, w, killed, "killed")
    y_kill = host(gpu_fwd(to_device(killed))[0])
    from tests.tolerances import within
    frac_changed = 1.0 - within(y_kill[:, 1:], y_sel[:, 1:], "bf16").mean()
    assert frac_changed > 0.5, frac_changed


def test_deterministic_replay():
    w = I.WORKLOADS["long"].with_(seqlen=8192, d_inner=256)
    d = to_device(I.make_inputs(w))
    a = [host_bits(t) for t in gpu_fwd(d)]
    b = [host_bits(t) for t in gpu_fwd(d)]
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_nonfinite_inputs_propagate(oracle):
    w = I.WORKLOADS["m130"].with_(batch=2, seqlen=40, d_inner=16, seed=13)
    inp = I.make_inputs(w)
    nan16 = I.f32_to_bf16_bits(np.array([np.nan], dtype=np.float32))[0]
    inp["xp"][1, 10, 5] = nan16
    inp["dt_raw"][0, 3, 2] = I.f32_to_bf16_bits(np.array([np.inf], dtype=np.float32))[0]
    y, h, cs = gpu_fwd(to_device(inp))
    yo, ho, _ = oracle_full(oracle, inp)
    yg, hg = host(y), host(h)
    fin = same_nonfinite_pattern(yg, yo, "y")
    assert_close(yg[fin], yo[fin], "bf16", "finite part of y")
    fin = same_nonfinite_pattern(hg, ho, "h")
    assert_close(hg[fin], ho[fin], "bf16", "finite part of h")


def test_guard_bands_untouched():
    """Outputs written exactly in their bounds: sentinels around each output survive."""
    w = I.WORKLOADS["long"].with_(batch=2, seqlen=3000, d_inner=72, seed=14)
    d = to_device(I.make_inputs(w))
    pad = 64
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    sent_bf16 = torch.tensor(-12288.0, dtype=torch.bfloat16)
    ybuf = torch.full((Bt * L * Di + 2 * pad,), sent_bf16.item(), dtype=torch.bfloat16, device="cuda")
    hbuf = torch.full((Bt * Di * N + 2 * pad,), -777.0, dtype=torch.float32, device="cuda")
    cbuf = torch.full((Bt * Di * 3 + 2 * pad,), sent_bf16.item(), dtype=torch.bfloat16, device="cuda")
    y = ybuf[pad:pad + Bt * L * Di].view(Bt, L, Di)
    h = hbuf[pad:pad + Bt * Di * N].view(Bt, Di, N)
    cs = cbuf[pad:pad + Bt * Di * 3].view(Bt, Di, 3)
    gpu_fwd(d, y=y, h_out=h, conv_state_out=cs)
    torch.cuda.synchronize()
    for buf, n, s in ((ybuf, Bt * L * Di, -12288.0), (hbuf, Bt * Di * N, -777.0),
                      (cbuf, Bt * Di * 3, -12288.0)):
        assert torch.all(buf[:pad].float() == s) and torch.all(buf[pad + n:].float() == s)
        assert not torch.any(buf[pad:pad + n].float() == s)


def test_runs_on_a_side_stream(oracle):
    w = I.WORKLOADS["m130"].with_(batch=2, seqlen=200, d_inner=64, seed=15)
    inp = I.make_inputs(w)
    d = to_device(inp)
    s = torch.cuda.Stream()
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        y, h, cs = gpu_fwd(d)
    s.synchronize()
    yo, ho, _ = oracle_full(oracle, inp)
    assert_close(host(y), yo, "bf16", "side stream")


def test_optional_state_outputs(oracle):
    w = I.WORKLOADS["tiny"]
    inp = I.make_inputs(w)
    y, h, cs = gpu_fwd(to_device(inp), want_states=False)
    assert h is None and cs is None
    yo, _, _ = oracle_full(oracle, inp)
    assert_close(host(y), yo, "f32", "no state outputs")
