"""GPU parity of the packed-document / initial-state forward (mamba_mixer_fwd_packed
through the C ABI) with the oracle (niverel-mamba 0.1.0, section "seq_idx strict reset").

The nine structural seq_idx cases of that section on a short multi-tile row, in fp32 and
bf16, with and without an initial state; the same at L = 8192 where the plan cuts the row
into 256-step time chunks, with boundaries on chunk edges; a long prompt fed in two calls
through (h, conv state); and the plain forward reproduced when the extras are absent.
"""

import numpy as np
import pytest
import torch

from selective_state_space_silu_b200 import inputs as I
from selective_state_space_silu_b200 import mixer as M
from tests.gpu_util import host, to_device
from tests.tolerances import assert_close

pytestmark = pytest.mark.gpu


def _inputs(Bt, L, Di, N, io, seed, state):
    w = I.Workload("packed", Bt, L, Di, N, 4, io, seed, decode=state)
    return w, I.make_inputs(w)


def _gpu(d, seq=None, h_in=None, cs_in=None):
    return M.mamba_mixer_fwd_packed(
        d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"], d["conv_w"],
        d.get("conv_b"), d["dt_bias"], seq_idx=seq, h_in=h_in, conv_state_in=cs_in)


def _oracle(oracle, inp, seq=None, state=False):
    w = I.as_f64
    return oracle.mixer(w(inp["xp"]), w(inp["z"]), w(inp["dt_raw"]), w(inp["B"]), w(inp["C"]),
                        inp["A_log"], inp["D"], inp["conv_w"], inp.get("conv_b"),
                        inp["dt_bias"], inp["h"] if state else None,
                        w(inp["conv_state"]) if state else None, nthreads=0, seq_idx=seq)


def _compare(oracle, w, inp, seq, state, what):
    d = to_device(inp)
    seq_d = None if seq is None else torch.from_numpy(seq).cuda()
    y, h, cs = _gpu(d, seq_d, d["h"] if state else None, d["conv_state"] if state else None)
    torch.cuda.synchronize()
    yo, ho, cso = _oracle(oracle, inp, seq, state)
    assert_close(host(y), yo, w.io_dtype, f"{what} y")
    assert_close(host(h), ho, w.io_dtype, f"{what} h_out")
    np.testing.assert_array_equal(host(cs), cso)   # a copy of inputs (or zeros): bitwise


@pytest.mark.parametrize("state", [False, True])
@pytest.mark.parametrize("io,N", [(I.F32, 16), (I.BF16, 16), (I.BF16, 8)])
@pytest.mark.parametrize("case", I.SEQ_IDX_CASES)
def test_nine_cases_short_rows(oracle, case, io, N, state):
    # 300 steps: ten 32-step tiles with a ragged tail; boundaries on tile edges (32)
    w, inp = _inputs(3, 300, 64, N, io, 2000 + I.SEQ_IDX_CASES.index(case), state)
    seq = I.seq_idx_case(case, 3, 300, edge=32, seed=7)
    _compare(oracle, w, inp, seq, state, f"{case} {io} N{N} state={state}")


@pytest.mark.parametrize("state", [False, True])
@pytest.mark.parametrize("case", ["boundary_on_edge", "many_short_docs", "misaligned_rows",
                                  "doc_inside_chunk", "terminal_padding"])
def test_chunked_rows_at_8192(oracle, case, state):
    w, inp = _inputs(2, 8192, 64, 16, I.BF16, 2100 + len(case), state)
    dims = M.make_dims(2, 8192, 64, 16, 4, M.MAMBA_BF16)
    plan = M.mamba_mixer_fwd_plan(dims)
    assert plan["nchunks"] > 1                              # the rows are cut into chunks
    # documents placed against the plan's chunk edges
    seq = I.seq_idx_case(case, 2, 8192, edge=plan["chunk_len"], seed=11)
    _compare(oracle, w, inp, seq, state, f"L8192 {case} state={state}")


def test_prompt_in_two_pieces(oracle):
    """fwd over x[:, :L1], then the rest from its (h, conv state): the second piece must
    match the oracle's full-sequence outputs for those steps."""
    w, inp = _inputs(2, 3000, 96, 16, I.BF16, 2200, False)
    d = to_device(inp)
    L1 = 1234
    first = {k: (v[:, :L1].contiguous() if k in ("xp", "z", "dt_raw", "B", "C") else v)
             for k, v in d.items()}
    rest = {k: (v[:, L1:].contiguous() if k in ("xp", "z", "dt_raw", "B", "C") else v)
            for k, v in d.items()}
    _, h1, cs1 = _gpu(first)
    y2, h2, cs2 = _gpu(rest, None, h1, cs1)
    torch.cuda.synchronize()
    yo, ho, cso = _oracle(oracle, inp)
    assert_close(host(y2), yo[:, L1:], w.io_dtype, "second piece y")
    assert_close(host(h2), ho, w.io_dtype, "second piece h_out")
    np.testing.assert_array_equal(host(cs2), cso)


@pytest.mark.parametrize("L", [1, 2, 3, 5])
def test_short_rows_with_initial_window(oracle, L):
    """L < 3: the returned conv state mixes the initial window and the new inputs."""
    w, inp = _inputs(2, L, 64, 16, I.BF16, 2300 + L, True)
    seq = np.zeros((2, L), dtype=np.int32)
    if L >= 2:
        seq[1, L - 1] = 1     # row 1: its last token is a document of its own
    _compare(oracle, w, inp, seq, True, f"L={L}")


def test_empty_sequence_returns_the_initial_state():
    w, inp = _inputs(2, 0, 64, 16, I.BF16, 2400, True)
    d = to_device(inp)
    y, h, cs = _gpu(d, None, d["h"], d["conv_state"])
    torch.cuda.synchronize()
    assert torch.equal(h, d["h"]) and torch.equal(cs, d["conv_state"])


def test_no_extras_is_the_plain_forward():
    from tests.gpu_util import gpu_fwd
    w, inp = _inputs(2, 700, 128, 16, I.BF16, 2500, False)
    d = to_device(inp)
    a = gpu_fwd(d)
    b = _gpu(d)
    torch.cuda.synchronize()
    assert all(torch.equal(u, v) for u, v in zip(a, b))


def test_constant_ids_match_the_plain_forward():
    from tests.gpu_util import gpu_fwd
    w, inp = _inputs(2, 700, 128, 16, I.BF16, 2501, False)
    d = to_device(inp)
    y0, h0, cs0 = gpu_fwd(d)
    y1, h1, cs1 = _gpu(d, torch.full((2, 700), 5, dtype=torch.int32, device="cuda"))
    torch.cuda.synchronize()
    assert_close(host(y1), host(y0), w.io_dtype, "constant ids y")
    assert_close(host(h1), host(h0), w.io_dtype, "constant ids h")
    assert torch.equal(cs0, cs1)
