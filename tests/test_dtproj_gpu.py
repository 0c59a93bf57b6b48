"""Parity of the forward with the dt projection fused (mamba_mixer_fwd_dtproj) against the
fp64 oracle (matmul, then the mixer): dt_raw = dt_low W_dt^T formed per tile on the tensor
cores.  Cases cover one and four time groups, chained chunks, two K blocks of dt_rank, a
dt_rank that is not a multiple of 16, d_state 8, ragged lengths and channel tiles, and the
130M-class layer in full on sampled channels."""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import host, pick_channels, to_device
from tests.tolerances import assert_close

pytestmark = pytest.mark.gpu


def _run(d):
    return M.mamba_mixer_fwd_dtproj(d["xp"], d["z"], d["dt_low"], d["W_dt"], d["B"], d["C"],
                                    d["A_log"], d["D"], d["conv_w"], d.get("conv_b"),
                                    d["dt_bias"])


def _dims(w):
    return M.make_dims(w.batch, w.seqlen, w.d_inner, w.d_state, 4, M.MAMBA_BF16)


@pytest.mark.parametrize("Bt,L,Di,N,R,groups", [
    (2, 300, 64, 16, 48, 4),       # four time groups, one chunk, ragged last tile
    (2, 4100, 96, 16, 80, 4),      # chained chunks, two K blocks of dt_rank
    (3, 77, 40, 8, 24, 4),         # d_state 8, dt_rank not a multiple of 16, ragged tile
    (10, 200, 1024, 16, 16, 1),    # 320 channel tiles: one time group
    (10, 65, 968, 16, 128, 1),     # one time group, ragged channel tile, dt_rank 128
    (10, 100, 1024, 8, 64, 1),     # one time group, d_state 8, one full K block
])
def test_dtproj_matches_oracle(oracle, Bt, L, Di, N, R, groups):
    w = I.Workload("dtproj", Bt, L, Di, N, 4, I.BF16, 5000 + L + R)
    plan = M.mamba_mixer_fwd_plan(_dims(w))
    inp = I.make_dtproj_inputs(w, R)
    y, h, cs = _run(to_device(inp))
    torch.cuda.synchronize()
    f = I.as_f64
    yo, ho, cso = oracle.mixer_dtproj(f(inp["xp"]), f(inp["z"]), f(inp["dt_low"]), f(inp["W_dt"]),
                                      f(inp["B"]), f(inp["C"]), inp["A_log"], inp["D"],
                                      inp["conv_w"], inp["conv_b"], inp["dt_bias"], nthreads=0)
    assert_close(host(y), yo, "bf16", f"dtproj y {Bt}x{L}x{Di} R{R}")
    assert_close(host(h), ho, "bf16", f"dtproj h {Bt}x{L}x{Di} R{R}")
    np.testing.assert_array_equal(host(cs), cso)
    if groups == 4:
        assert plan["time_groups"] == 4


def test_dtproj_m130_sampled(oracle):
    """The 130M-class layer (8 x 2048 x 1536, dt_rank 48 = d_model / 16) on sampled channels."""
    w = I.WORKLOADS["m130"]
    inp = I.make_dtproj_inputs(w, 48)
    y, h, cs = _run(to_device(inp))
    torch.cuda.synchronize()
    bi = np.arange(w.batch)
    di = pick_channels(w.d_inner, 48, 9)
    yo, ho, cso = oracle.mixer_dtproj_channels(inp, bi, di, nthreads=0, widen=I.as_f64)
    idx = torch.as_tensor(di, device="cuda")
    assert_close(host(y[:, :, idx]), yo, "bf16", "dtproj m130 y (sampled)")
    assert_close(host(h)[:, di], ho, "bf16", "dtproj m130 h (sampled)")
    np.testing.assert_array_equal(host(cs)[:, di], cso)


def test_dtproj_rejects_unsupported_ranks():
    w = I.Workload("dtproj_bad", 1, 64, 64, 16, 4, I.BF16, 5100)
    inp = I.make_dtproj_inputs(w, 20)               # not a multiple of 8
    with pytest.raises(M.MambaError) as e:
        _run(to_device(inp))
    assert e.value.code == 2
