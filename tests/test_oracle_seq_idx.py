"""Pins for the oracle's packed-document reset (niverel-mamba 0.1.0, section "seq_idx
strict reset"): a row with seq_idx must equal its documents run one by one and
concatenated, with both the conv state and the SSM state starting from zero at every
document after the first.  The documents are run through the oracle without seq_idx, the
path pinned by test_oracle_pins.py, so a wrong reset (a missed conv tap, a state carried
across a boundary, a reset one step late, the wrong final states) fails here.
"""

import numpy as np
import pytest

from selective_state_space_silu_b200 import inputs as I
from tests.test_oracle_pins import rand_case, run


def doc_runs(row):
    """(start, end) of the maximal runs of equal ids in one row."""
    cuts = [0] + [t for t in range(1, len(row)) if row[t] != row[t - 1]] + [len(row)]
    return list(zip(cuts[:-1], cuts[1:]))


def concat_of_documents(oracle, c, seq):
    """Each row split at its id changes, every document run alone, outputs concatenated;
    the row's initial state (if any) goes to its first document only."""
    Bt, L, Di = c["xp"].shape
    y = np.empty((Bt, L, Di))
    h = np.empty(c["h_in"].shape if c.get("h_in") is not None else (Bt, Di, c["A_log"].shape[1]))
    cs = np.empty((Bt, Di, c["conv_w"].shape[1] - 1))
    for b in range(Bt):
        for k, (s, e) in enumerate(doc_runs(seq[b])):
            sub = dict(c)
            for name in ("xp", "z", "dt_raw", "B", "C"):
                sub[name] = c[name][b:b + 1, s:e]
            first = k == 0
            sub["h_in"] = c["h_in"][b:b + 1] if first and c.get("h_in") is not None else None
            sub["conv_state_in"] = (c["conv_state_in"][b:b + 1]
                                    if first and c.get("conv_state_in") is not None else None)
            yd, hd, csd = run(oracle, sub)
            y[b, s:e] = yd[0]
            h[b], cs[b] = hd[0], csd[0]
    return y, h, cs


@pytest.mark.parametrize("state", [False, True])
@pytest.mark.parametrize("case", I.SEQ_IDX_CASES)
def test_packed_row_equals_documents_run_alone(oracle, case, state):
    c = rand_case(50 + I.SEQ_IDX_CASES.index(case), Bt=3, L=24, Di=3, N=3, state=state)
    seq = I.seq_idx_case(case, 3, 24, edge=8, seed=5)
    y, h, cs = run(oracle, c, seq_idx=seq)
    ye, he, cse = concat_of_documents(oracle, c, seq)
    # the same operations in the same order: equal to the last bit
    assert np.array_equal(y, ye) and np.array_equal(h, he) and np.array_equal(cs, cse)


def test_constant_ids_change_nothing(oracle):
    c = rand_case(70, Bt=2, L=20, Di=3, N=4, state=True)
    seq = np.full((2, 20), 9, dtype=np.int32)
    a, b = run(oracle, c, seq_idx=seq), run(oracle, c)
    assert all(np.array_equal(u, v) for u, v in zip(a, b))


def test_resets_do_change_the_outputs(oracle):
    """Control: a boundary must act (outputs after it differ from the unpacked run), while
    outputs before the first boundary stay equal (causality)."""
    c = rand_case(71, Bt=1, L=30, Di=4, N=4)
    seq = I.seq_idx_case("doc_inside_chunk", 1, 30)
    first = doc_runs(seq[0])[1][0]
    y1, _, _ = run(oracle, c, seq_idx=seq)
    y0, _, _ = run(oracle, c)
    assert np.array_equal(y1[:, :first], y0[:, :first])
    assert np.abs(y1[:, first:first + 4] - y0[:, first:first + 4]).max() > 1e-3


def test_conv_state_out_is_the_last_documents(oracle):
    """A last document shorter than the conv window leaves zeros in the older slots of
    the returned conv state, as if it had been run alone from zero."""
    c = rand_case(72, Bt=1, L=12, Di=2, N=3, state=True)
    seq = np.array([[0] * 10 + [1] * 2], dtype=np.int32)
    _, _, cs = run(oracle, c, seq_idx=seq)
    np.testing.assert_array_equal(cs[0, :, 0], 0.0)
    np.testing.assert_array_equal(cs[0, :, 1:], c["xp"][0, 10:12].T)
