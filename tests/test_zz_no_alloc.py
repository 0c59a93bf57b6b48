"""The forward for callers that cannot allocate device memory (mamba_mixer_fwd_noalloc).

Plugin hosts that hand over only input and output buffers, code running inside an
allocator's callback, and latency-critical paths that must avoid cudaMalloc's device-wide
synchronisation cannot give mamba_mixer_fwd the workspace it asks for.  The no-alloc entry
point serves them from a fixed 2 MiB scratch array inside the library.  These tests call it
through the C ABI and check that two calls in a row give what mamba_mixer_fwd gives (and what
the oracle gives), within the tolerance the other GPU tests use, also when a call on other
sizes runs in between; that its status check reports a bounded-wait timeout; and that sizes
needing more scratch are refused.  This file is collected last on purpose.
"""

import ctypes

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import build as Bld
from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import gpu_fwd, host, host_bits, oracle_full, to_device
from tests.tolerances import assert_close


def _noalloc(d):
    return M.mamba_mixer_fwd_noalloc(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"],
                                     d["D"], d["conv_w"], d.get("conv_b"), d["dt_bias"])


def _dims(w):
    return M.make_dims(w.batch, w.seqlen, w.d_inner, w.d_state, 4,
                       M.MAMBA_BF16 if w.io_dtype == "bf16" else M.MAMBA_F32)


@pytest.mark.gpu
@pytest.mark.parametrize("w", [
    # long enough to be cut into time chunks, so the scratch carries the chunk aggregates
    I.Workload("noalloc_bf16", 2, 4096, 128, 16, 4, "bf16", 2024),
    I.Workload("noalloc_f32", 2, 1500, 64, 8, 4, "f32", 2025),
], ids=lambda w: w.name)
def test_noalloc_matches_fwd_on_two_calls(w, oracle):
    Bld.build()
    assert M.mamba_mixer_fwd_workspace_bytes(_dims(w)) > 256   # the scratch is really used
    # a call on other inputs and a different chunk count, run between the checked calls:
    # the checked call must not read aggregates this one left in the shared scratch
    # (its wider d_inner puts every aggregate of it at another place in the scratch)
    other = w.with_(seqlen=w.seqlen // 2 + 96, d_inner=w.d_inner + 64, seed=w.seed + 100)
    assert M.mamba_mixer_fwd_workspace_bytes(_dims(other)) > 256
    inp = I.make_inputs(w)
    d = to_device(inp)
    d_other = to_device(I.make_inputs(other))
    y0, h0, c0 = gpu_fwd(d)
    yo, ho, _ = oracle_full(oracle, inp)
    for call in range(2):
        if call == 1:
            _noalloc(d_other)
        y, h, cs = _noalloc(d)
        torch.cuda.synchronize()
        M.mamba_mixer_noalloc_check()
        assert_close(host(y), host(y0), w.io_dtype, f"no-alloc y vs mamba_mixer_fwd, call {call + 1}")
        assert_close(host(h), host(h0), w.io_dtype, f"no-alloc h_out vs mamba_mixer_fwd, call {call + 1}")
        np.testing.assert_array_equal(host_bits(cs), host_bits(c0))
        assert_close(host(y), yo, w.io_dtype, f"no-alloc y vs oracle, call {call + 1}")
        assert_close(host(h), ho, w.io_dtype, f"no-alloc h_out vs oracle, call {call + 1}")


@pytest.mark.gpu
def test_noalloc_check_reports_a_bounded_wait_timeout(oracle):
    """A wait that runs out (the library's test-only injection: one CTA arms a tile's barrier
    but issues none of its copies) is reported by mamba_mixer_noalloc_check, which clears
    it; the next call on the same scratch is correct again.  No GPU fault is involved."""
    Bld.build()
    w = I.Workload("noalloc_fail", 1, 300, 64, 16, 4, "bf16", 78)
    assert M.mamba_mixer_fwd_launches(_dims(w)) == 1
    inp = I.make_inputs(w)
    d = to_device(inp)
    M.mamba_mixer_noalloc_check()                      # start from a clear status word
    M.mamba_mixer_set_fault_injection(1)              # read by the host at launch
    try:
        _noalloc(d)
    finally:
        M.mamba_mixer_set_fault_injection(-1)
    with pytest.raises(M.MambaError) as err:
        M.mamba_mixer_noalloc_check()
    assert err.value.code == 6 and "bounded wait" in str(err.value)
    M.mamba_mixer_noalloc_check()                      # the check cleared it
    y, h, _ = _noalloc(d)
    M.mamba_mixer_noalloc_check()
    yo, ho, _ = oracle_full(oracle, inp)
    assert_close(host(y), yo, "bf16", "y after a timed-out no-alloc call")
    assert_close(host(h), ho, "bf16", "h after a timed-out no-alloc call")


def test_noalloc_refuses_sizes_beyond_its_scratch():
    """Sizes whose forward needs more than the fixed 2 MiB of scratch are refused before any
    CUDA call, with the reason in mamba_last_error.  (The dims are searched for, since the
    scratch a forward needs depends on how the library splits long sequences.)"""
    Bld.build()
    lib = M.load_library()
    lib.mamba_mixer_fwd_noalloc.restype = ctypes.c_int
    lib.mamba_mixer_fwd_noalloc.argtypes = [ctypes.POINTER(M.mamba_dims)] + [ctypes.c_void_p] * 14
    dims = None
    for io in (M.MAMBA_BF16, M.MAMBA_F32):
        for Di in range(256, 65536, 256):
            cand = M.make_dims(1, 1 << 20, Di, 16, 4, io)
            if M.mamba_mixer_fwd_workspace_bytes(cand) > (2 << 20):
                dims = cand
                break
        if dims is not None:
            break
    assert dims is not None, "no size exceeds the scratch: the refusal path would be dead"
    fake = [ctypes.c_void_p(0x10000000 + i * (1 << 36)) for i in range(13)]
    rc = lib.mamba_mixer_fwd_noalloc(ctypes.byref(dims), *fake, None)
    assert rc == 4, M.mamba_last_error()
    assert "scratch" in M.mamba_last_error()
