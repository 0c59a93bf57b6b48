"""Failure detection without a GPU fault: a bounded wait that runs out.

The forward kernel waits on its own asynchronous copies through mbarriers; every wait gives
up after one second, stops the CTA cleanly and records MAMBA_ERR_TIMEOUT in the workspace
status word, which mamba_mixer_check reports and clears.  The test makes one wait run out
with the library's test-only injection (one CTA arms a tile's barrier but issues none of its
copies), checks the reported status, then checks that the same context still computes
correct results.  Nothing here faults, traps or hangs the GPU.
"""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import gpu_fwd, host, oracle_full, to_device
from tests.tolerances import assert_close

pytestmark = pytest.mark.gpu


def test_bounded_wait_reports_timeout_and_context_survives(oracle):
    w = I.Workload("fail", 1, 300, 64, 16, 4, "bf16", 77)      # one kernel, 10 tiles
    inp = I.make_inputs(w)
    d = to_device(inp)
    dims = M.make_dims(w.batch, w.seqlen, w.d_inner, w.d_state, 4, M.MAMBA_BF16)
    assert M.mamba_mixer_fwd_launches(dims) == 1
    ws = M.new_workspace(dims, "cuda")

    M.mamba_mixer_set_fault_injection(1)   # read by the host when it builds the launch
    try:
        gpu_fwd(d, workspace=ws)
    finally:
        M.mamba_mixer_set_fault_injection(-1)
    with pytest.raises(M.MambaError) as err:
        M.mamba_mixer_check(ws)
    assert err.value.code == 6 and "bounded wait" in str(err.value)
    M.mamba_mixer_check(ws)            # the check cleared the status word

    y, h, cs = gpu_fwd(d, workspace=ws)
    M.mamba_mixer_check(ws)            # clean run: no error
    torch.cuda.synchronize()
    yo, ho, cso = oracle_full(oracle, inp)
    assert_close(host(y), yo, "bf16", "y after a timed-out launch")
    assert_close(host(h), ho, "bf16", "h after a timed-out launch")
    np.testing.assert_array_equal(host(cs), cso)
