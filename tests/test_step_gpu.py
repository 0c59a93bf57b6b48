"""GPU parity of the decode step (mamba_mixer_step through the C ABI) with the oracle,
and the decode contract: prefill-then-step equals a full forward (niverel-mamba 0.1.0,
section "Autoregressive decoding"), functional by default, in place on request."""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import gpu_fwd, gpu_step, host, host_bits, oracle_full, to_device
from tests.tolerances import assert_close

pytestmark = pytest.mark.gpu


def _check_step(oracle, w, inp=None, what=""):
    inp = inp if inp is not None else I.make_inputs(w)
    d = to_device(inp)
    y, h, cs = gpu_step(d, d["h"], d["conv_state"])
    torch.cuda.synchronize()
    yo, ho, cso = oracle_full(oracle, inp, with_state=True)
    assert_close(host(y), yo, w.io_dtype, f"{what or w.name} y")
    assert_close(host(h), ho, w.io_dtype, f"{what or w.name} h_out")
    np.testing.assert_array_equal(host(cs), cso)


def test_decode_full_size(oracle):
    """256 sequences x 5120 channels, every output checked."""
    _check_step(oracle, I.WORKLOADS["decode"])


@pytest.mark.parametrize("io,N", [("f32", 16), ("f32", 8), ("bf16", 8)])
def test_decode_dtypes_and_states(oracle, io, N):
    w = I.Workload("dec", 6, 1, 136, N, 4, io, 300 + N, decode=True)
    _check_step(oracle, w, what=f"{io} N={N}")


def test_decode_no_conv_bias_random_params(oracle):
    w = I.WORKLOADS["decode"].with_(batch=8, d_inner=256)
    inp = I.make_inputs(w)
    inp.update(I.random_params(w, 5))
    inp["conv_b"] = None
    _check_step(oracle, w, inp, "random params")


def test_functional_inputs_untouched():
    w = I.WORKLOADS["decode"].with_(batch=16, d_inner=512)
    d = to_device(I.make_inputs(w))
    h0 = d["h"].clone()
    c0 = d["conv_state"].clone()
    gpu_step(d, d["h"], d["conv_state"])
    torch.cuda.synchronize()
    assert torch.equal(d["h"], h0) and torch.equal(d["conv_state"], c0)


def test_in_place_matches_functional():
    w = I.WORKLOADS["decode"].with_(batch=32, d_inner=1024)
    d = to_device(I.make_inputs(w))
    y1, h1, c1 = gpu_step(d, d["h"], d["conv_state"])
    h = d["h"].clone()
    c = d["conv_state"].clone()
    y2, h2, c2 = gpu_step(d, h, c, h_out=h, conv_state_out=c)
    torch.cuda.synchronize()
    assert h2.data_ptr() == h.data_ptr()
    np.testing.assert_array_equal(host_bits(y1), host_bits(y2))
    np.testing.assert_array_equal(host_bits(h1), host_bits(h))
    np.testing.assert_array_equal(host_bits(c1), host_bits(c))


@pytest.mark.parametrize("io,L,k", [("bf16", 64, 5), ("f32", 32, 7), ("bf16", 3000, 3),
                                    ("bf16", 2, 2)])
def test_prefill_then_steps_equals_forward(oracle, io, L, k):
    """GPU forward over the first L-k tokens, then k GPU decode steps, reproduces the
    oracle's forward over all L tokens (y for every token, final h and conv state)."""
    w = I.Workload("pf", 2, L, 128, 16, 4, io, 400 + L)
    inp = I.make_inputs(w)
    d = to_device(inp)
    pre = {key: (v[:, : L - k].contiguous() if key in ("xp", "z", "dt_raw", "B", "C") else v)
           for key, v in d.items()}
    yp, h, cs = gpu_fwd(pre)
    ys = [yp]
    for t in range(L - k, L):
        st = {key: (v[:, t: t + 1].contiguous() if key in ("xp", "z", "dt_raw", "B", "C") else v)
              for key, v in d.items()}
        yt, h, cs = gpu_step(st, h, cs, h_out=h, conv_state_out=cs)
        ys.append(yt)
    y = torch.cat(ys, dim=1)
    torch.cuda.synchronize()
    yo, ho, cso = oracle_full(oracle, inp)
    assert_close(host(y), yo, io, "prefill+steps y")
    assert_close(host(h), ho, io, "prefill+steps h")
    np.testing.assert_array_equal(host(cs), cso)
    yf, hf, csf = gpu_fwd(d)
    np.testing.assert_array_equal(host_bits(csf), host_bits(cs))


def test_steps_from_zero_state_equal_forward(oracle):
    w = I.Workload("z0", 4, 12, 64, 16, 4, "bf16", 501)
    inp = I.make_inputs(w)
    d = to_device(inp)
    h = torch.zeros((4, 64, 16), dtype=torch.float32, device="cuda")
    cs = torch.zeros((4, 64, 3), dtype=torch.bfloat16, device="cuda")
    ys = []
    for t in range(12):
        st = {key: (v[:, t: t + 1].contiguous() if key in ("xp", "z", "dt_raw", "B", "C") else v)
              for key, v in d.items()}
        yt, h, cs = gpu_step(st, h, cs)
        ys.append(yt)
    yo, ho, _ = oracle_full(oracle, inp)
    assert_close(host(torch.cat(ys, 1)), yo, "bf16", "steps from zero")
    assert_close(host(h), ho, "bf16", "steps from zero h")



def test_decode_unaligned_conv_state(oracle):
    """A conv state 2 bytes off a 16-byte boundary (the API allows 2-byte alignment)."""
    w = I.Workload("dec_u", 5, 1, 200, 16, 4, "bf16", 321, decode=True)
    inp = I.make_inputs(w)
    d = to_device(inp)
    n = d["conv_state"].numel()
    buf = torch.empty(n + 8, dtype=d["conv_state"].dtype, device="cuda")
    cs_in = buf[1:1 + n].view(d["conv_state"].shape)
    cs_in.copy_(d["conv_state"])
    assert cs_in.data_ptr() % 16 != 0
    y, h, cs = gpu_step(d, d["h"], cs_in)
    torch.cuda.synchronize()
    yo, ho, cso = oracle_full(oracle, inp, with_state=True)
    assert_close(host(y), yo, w.io_dtype, "unaligned y")
    assert_close(host(h), ho, w.io_dtype, "unaligned h_out")
    np.testing.assert_array_equal(host(cs), cso)


def test_step_status_word_is_clear_after_clean_steps(oracle):
    """The step reports bounded-wait timeouts through its own status word (it takes no
    workspace); after ordinary steps mamba_mixer_step_check finds it clear."""
    w = I.WORKLOADS["decode"].with_(batch=5, d_inner=200, seed=4242)
    inp = I.make_inputs(w)
    d = to_device(inp)
    for _ in range(2):
        gpu_step(d, d["h"], d["conv_state"])
    M.mamba_mixer_step_check()
