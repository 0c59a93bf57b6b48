"""Host-side checks of mamba2_ssd_fwd: argument validation before anything is enqueued.

Nothing here launches a kernel: every call fails validation (before the first CUDA call)
or has nothing to do (batch 0 or nheads 0).
"""

import ctypes

import pytest

from selective_state_space_silu_b200 import build as Bld
from selective_state_space_silu_b200 import mixer as M
from selective_state_space_silu_b200 import ssd as S

NAMES = ["x", "dt", "A_log", "B", "C", "D", "dt_bias", "z", "seq", "h_in", "y", "h_out"]


@pytest.fixture(scope="module")
def lib():
    Bld.build()
    return S._lib()


def _fake(addr):
    return ctypes.c_void_p(addr)


def _call(lib, dims, ptrs=None):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(NAMES)}
    if ptrs:
        p.update(ptrs)
    ws = p.get("ws", _fake(0xf000000000))
    ws_bytes = p.get("ws_bytes", 1 << 40)
    return lib.mamba2_ssd_fwd(ctypes.byref(dims) if dims is not None else None,
                              *[p[k] for k in NAMES], ws, ws_bytes, None)


def dims(**kw):
    a = dict(batch=2, seqlen=100, nheads=4, headdim=64, d_state=128, ngroups=1,
             io_dtype=M.MAMBA_BF16)
    a.update(kw)
    return S.make_dims(**a)


def test_unsupported_and_invalid_dims(lib):
    for kw, code in [(dict(io_dtype=M.MAMBA_F32), 2), (dict(headdim=32), 2),
                     (dict(d_state=16), 2), (dict(d_state=256), 2), (dict(batch=70000), 2),
                     (dict(ngroups=3), 1), (dict(ngroups=0), 1), (dict(seqlen=-1), 1),
                     (dict(nheads=-4), 1)]:
        rc = _call(lib, dims(**kw))
        assert rc == code, (kw, rc, M.mamba_last_error())
        assert M.mamba_last_error()


def test_null_dims_and_reserved(lib):
    assert _call(lib, None) == 1
    d = dims()
    d.reserved = 5
    assert _call(lib, d) == 1
    assert "reserved" in M.mamba_last_error()


def test_null_required_pointers(lib):
    for k in ("x", "dt", "A_log", "B", "C", "D", "dt_bias", "y"):
        assert _call(lib, dims(), {k: None}) == 1, k
        assert k.replace("dt", "dt_raw") in M.mamba_last_error() or k in M.mamba_last_error()


def test_misaligned_pointers(lib):
    assert _call(lib, dims(), {"x": _fake(0x10000008)}) == 3
    assert _call(lib, dims(), {"B": _fake(0x3010000004)}) == 3
    assert _call(lib, dims(), {"dt": _fake(0x1010000001)}) == 3
    assert _call(lib, dims(), {"D": _fake(0x5010000002)}) == 3
    assert _call(lib, dims(), {"h_out": _fake(0xb010000008)}) == 3
    assert _call(lib, dims(), {"seq": _fake(0x8010000002)}) == 3


def test_overlaps_rejected(lib):
    assert _call(lib, dims(), {"y": _fake(0x10000000)}) == 1            # y on top of x
    assert _call(lib, dims(), {"h_out": _fake(0xa010000000)}) == 1      # h_out inside y
    assert _call(lib, dims(), {"y": _fake(0x8010000000)}) == 1          # y on top of seq_idx
    # h_out == h_in exactly is in-place and allowed at validation; partial overlap is not
    assert _call(lib, dims(), {"h_out": _fake(0x9010000010)}) == 1
    assert "partially" in M.mamba_last_error()


def test_nothing_to_do(lib):
    assert _call(lib, dims(batch=0)) == 0
    assert _call(lib, dims(nheads=0), {k: None for k in ("A_log", "D", "dt_bias")}) == 0


def test_workspace_rules(lib):
    # few (row, head) pairs and a long sequence: split into time segments, workspace needed
    d = dims(batch=1, seqlen=8192, nheads=2)
    need = lib.mamba2_ssd_fwd_workspace_bytes(ctypes.byref(d))
    assert need > 0
    assert _call(lib, d, {"ws": None, "ws_bytes": 0}) == 4
    assert _call(lib, d, {"ws_bytes": need - 1}) == 4
    assert _call(lib, d, {"ws": _fake(0xf000000080), "ws_bytes": need}) == 3
    assert _call(lib, d, {"ws": _fake(0x10000000), "ws_bytes": need}) == 1   # overlaps x
    # many pairs: one segment, no workspace
    d = dims(batch=64, seqlen=256, nheads=24)
    assert lib.mamba2_ssd_fwd_workspace_bytes(ctypes.byref(d)) == 0
    assert lib.mamba2_ssd_fwd_workspace_bytes(ctypes.byref(dims(headdim=32))) == 0
    # size: per (row, head), segments - 1 end states and one copy of h_in (headdim x
    # d_state fp32 each), then segments - 1 floats, padded to 256 bytes
    d = dims(batch=2, seqlen=8192, nheads=24, d_state=128)
    need = lib.mamba2_ssd_fwd_workspace_bytes(ctypes.byref(d))
    nseg = need // (48 * 64 * 128 * 4)
    assert nseg >= 2
    assert need == 48 * nseg * 64 * 128 * 4 + (48 * (nseg - 1) * 4 + 255) // 256 * 256


def _nseg(lib, **kw):
    d = dims(**kw)
    need = lib.mamba2_ssd_fwd_workspace_bytes(ctypes.byref(d))
    if need == 0:
        return 1
    pairs = d.batch * d.nheads
    return need // (pairs * 64 * d.d_state * 4)


def test_segment_plan(lib):
    # the plan minimises the modelled time of the tensor-core passes: main-pass waves (one CTA
    # per SM, 148 SMs) x (5.3 + chunks per segment) x 1.675 us plus state-pass waves (two CTAs
    # per SM) x chunks per segment x 1.5 us, fewest segments on a tie
    assert _nseg(lib, batch=8, seqlen=2048, nheads=24) == 1       # 192 pairs: 2 waves, no state pass
    assert _nseg(lib, batch=2, seqlen=8192, nheads=24) == 6
    assert _nseg(lib, batch=1, seqlen=640, nheads=2) == 10        # 10 chunks, one each
    assert _nseg(lib, batch=1, seqlen=65536, nheads=2) == 16      # at most 16
    assert _nseg(lib, batch=64, seqlen=4096, nheads=24) == 1      # pairs fill the GPU
    assert _nseg(lib, batch=1, seqlen=64, nheads=4) == 1          # one chunk


STEP = ["x", "dt", "A_log", "B", "C", "D", "dt_bias", "z", "h_in", "y", "h_out"]


def _step(lib, d, ptrs=None):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(STEP)}
    if ptrs:
        p.update(ptrs)
    return lib.mamba2_ssd_step(ctypes.byref(d), *[p[k] for k in STEP], None)


def test_step_validation(lib):
    assert _step(lib, dims(seqlen=2)) == 1
    assert "one token" in M.mamba_last_error()
    for k in ("x", "dt", "B", "C", "h_in", "y", "h_out"):
        assert _step(lib, dims(seqlen=1), {k: None}) == 1, k
    assert _step(lib, dims(seqlen=1, d_state=16)) == 2
    assert _step(lib, dims(seqlen=1), {"h_in": _fake(0x8010000008)}) == 3
    # a partial overlap of the states is rejected (exact aliasing, in place, is allowed:
    # it passes validation, so it is exercised only by the GPU tests, never with fake pointers)
    assert _step(lib, dims(seqlen=1), {"h_out": _fake(0x8010000100)}) == 1
    assert _step(lib, dims(seqlen=1), {"y": _fake(0x10000000)}) == 1      # y on x
    assert _step(lib, dims(seqlen=1, batch=0)) == 0


CONV = ["xbc", "w", "bias", "seq", "cs_in", "x", "B", "C", "cs_out"]


def _conv(lib, d, ptrs=None):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(CONV)}
    if ptrs:
        p.update(ptrs)
    return lib.mamba2_conv_silu(ctypes.byref(d), *[p[k] for k in CONV], None)


def test_conv_validation(lib):
    assert _conv(lib, dims(), {"xbc": None}) == 1
    assert _conv(lib, dims(), {"x": None}) == 1
    assert _conv(lib, dims(), {"w": _fake(0x1010000008)}) == 3          # conv_w needs 16 bytes
    assert _conv(lib, dims(), {"B": _fake(0x6010000002)}) == 3
    assert _conv(lib, dims(), {"x": _fake(0x10000000)}) == 1            # x on top of xbc
    assert _conv(lib, dims(), {"C": _fake(0x6010000000)}) == 1          # C on top of B
    assert _conv(lib, dims(headdim=32)) == 2
    assert _conv(lib, dims(batch=0)) == 0


def _norm(lib, d, eps=1e-5, ptrs=None):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(["y", "z", "w", "out"])}
    if ptrs:
        p.update(ptrs)
    return lib.mamba2_gated_rmsnorm(ctypes.byref(d), p["y"], p["z"], p["w"], ctypes.c_float(eps),
                                    p["out"], None)


def test_norm_validation(lib):
    assert _norm(lib, dims(), eps=-1.0) == 1
    assert _norm(lib, dims(), eps=float("nan")) == 1
    assert _norm(lib, dims(), ptrs={"z": None}) == 1
    assert _norm(lib, dims(), ptrs={"w": _fake(0x2010000004)}) == 3
    assert _norm(lib, dims(), ptrs={"out": _fake(0x10000000)}) == 1    # out on top of y
    assert _norm(lib, dims(ngroups=3)) == 1                             # 4 heads, 3 groups
    assert _norm(lib, dims(seqlen=0)) == 0
