"""Host-side checks of the C ABI: the library loads, exports what include/*.h declares,
links no vendor math library, and rejects bad arguments before touching CUDA.

Nothing here launches a kernel: every call either fails validation (which happens before
the first CUDA call) or has nothing to do (batch 0).
"""

import ctypes
import glob
import os
import re
import subprocess

import pytest

from selective_state_space_silu_b200 import build as B
from selective_state_space_silu_b200 import mixer as M
from selective_state_space_silu_b200 import ssd as SSD

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return M.load_library()


def declared_symbols():
    names = set()
    for h in glob.glob(os.path.join(ROOT, "include", "*.h")):
        src = open(h).read()
        names |= set(re.findall(r"MAMBA_API\s+[\w\s\*]+?\b(mamba2?_\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol(lib):
    names = declared_symbols()
    assert set(M.EXPORTS) <= names
    assert set(SSD.EXPORTS) <= names
    out = subprocess.run(["nm", "-D", "--defined-only", M.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\sT\s(mamba2?_\w+)", out))
    assert names <= exported, names - exported
    for n in names:
        assert hasattr(lib, n)


def test_linkage_has_no_vendor_math_or_torch(lib):
    """No cuBLAS / cuDNN / libtorch, and the CUDA runtime is linked statically."""
    out = subprocess.run(["ldd", M.LIB_PATH], capture_output=True, text=True, check=True).stdout
    names = [line.split()[0].lower() for line in out.splitlines() if line.strip()]
    for bad in ("cublas", "cudnn", "torch", "c10", "cudart", "nccl", "cufft", "curand"):
        assert not any(bad in n for n in names), out


def test_version(lib):
    assert M.mamba_version().startswith("mamba_mixer ")


def _fake(addr):
    return ctypes.c_void_p(addr)


def _fwd(lib, dims, ptrs=None, ws=None, ws_bytes=0):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(
        ["xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias", "y", "h", "cs"])}
    if ptrs:
        p.update(ptrs)
    return lib.mamba_mixer_fwd(ctypes.byref(dims), p["xp"], p["z"], p["dt"], p["B"], p["C"],
                               p["A_log"], p["D"], p["conv_w"], p["conv_b"], p["dt_bias"],
                               p["y"], p["h"], p["cs"], ws, ws_bytes, None)


def _step(lib, dims, ptrs=None):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(
        ["xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias", "h_in", "cs_in",
         "y", "h", "cs"])}
    if ptrs:
        p.update(ptrs)
    return lib.mamba_mixer_step(ctypes.byref(dims), p["xp"], p["z"], p["dt"], p["B"], p["C"],
                                p["A_log"], p["D"], p["conv_w"], p["conv_b"], p["dt_bias"],
                                p["h_in"], p["cs_in"], p["y"], p["h"], p["cs"], None)


def test_unsupported_dims(lib):
    for kw, code in [(dict(d_conv=3), 2), (dict(d_state=32), 2), (dict(d_state=12), 2),
                     (dict(d_inner=12), 2), (dict(io_dtype=7), 2), (dict(batch=-1), 1),
                     (dict(seqlen=-5), 1)]:
        args = dict(batch=2, seqlen=16, d_inner=128, d_state=16, d_conv=4, io_dtype=M.MAMBA_BF16)
        args.update(kw)
        dims = M.make_dims(**args)
        rc = _fwd(lib, dims)
        assert rc == code, (kw, rc, M.mamba_last_error())
        assert M.mamba_last_error()
        assert lib.mamba_mixer_fwd_workspace_bytes(ctypes.byref(dims)) == 0


def test_reserved_and_null_dims(lib):
    d = M.make_dims(2, 16, 128, 16)
    d.reserved = 1
    assert _fwd(lib, d) == 1
    assert lib.mamba_mixer_fwd(None, *([None] * 13), None, 0, None) == 1
    assert "dims" in M.mamba_last_error()


def test_null_required_pointers(lib):
    dims = M.make_dims(2, 16, 128, 16)
    for k in ("xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "dt_bias", "y"):
        assert _fwd(lib, dims, {k: None}) == 1, k
    sd = M.make_dims(4, 1, 64, 16)
    for k in ("xp", "h_in", "cs_in", "h", "cs", "y"):
        assert _step(lib, sd, {k: None}) == 1, k


def test_misaligned_pointers(lib):
    dims = M.make_dims(2, 16, 128, 16)
    assert _fwd(lib, dims, {"xp": _fake(0x10000008)}) == 3
    assert "xp" in M.mamba_last_error()
    assert _fwd(lib, dims, {"D": _fake(0x6010000002)}) == 3
    sd = M.make_dims(4, 1, 64, 16)
    assert _step(lib, sd, {"h_in": _fake(0xa010000004)}) == 3


def test_overlaps_rejected(lib):
    dims = M.make_dims(2, 16, 128, 16)
    assert _fwd(lib, dims, {"y": _fake(0x10000000)}) == 1          # y on top of xp
    assert _fwd(lib, dims, {"h": _fake(0xa010000010)}) == 1          # h_out inside y
    sd = M.make_dims(4, 1, 64, 16)
    # exact in-place aliasing of the states is fine at validation; partial overlap is not
    assert _step(lib, sd, {"h": _fake(0xa010000040)}) == 1
    assert "partially" in M.mamba_last_error()
    assert _step(lib, sd, {"cs": _fake(0xb010000006)}) == 1
    assert _step(lib, M.make_dims(4, 2, 64, 16)) == 1               # step needs seqlen 1


def test_workspace_rules(lib):
    short = M.make_dims(8, 512, 1536, 16)
    assert lib.mamba_mixer_fwd_workspace_bytes(ctypes.byref(short)) == 256   # status header only
    assert lib.mamba_mixer_fwd_launches(ctypes.byref(short)) == 1
    assert _fwd(lib, short) == 4                                          # workspace required
    long = M.make_dims(2, 65536, 2560, 16)
    assert M.mamba_mixer_fwd_plan(long)["nchunks"] > 1
    need = lib.mamba_mixer_fwd_workspace_bytes(ctypes.byref(long))
    assert need > 0 and need % 16 == 0
    assert _fwd(lib, long) == 4
    assert "workspace" in M.mamba_last_error()
    assert _fwd(lib, long, ws=_fake(0x14010000000), ws_bytes=need - 16) == 4
    assert _fwd(lib, long, ws=_fake(0x14010000008), ws_bytes=need) == 4


def test_empty_batch_is_a_no_op(lib):
    d = M.make_dims(0, 16, 128, 16)
    ws = _fake(0x10000000 + 30 * (1 << 36))
    assert _fwd(lib, d, {k: None for k in ("xp", "z", "dt", "B", "C", "y", "h", "cs")},
                ws=ws, ws_bytes=256) == 0
    assert M.mamba_last_error() == ""
    assert lib.mamba_mixer_fwd_launches(ctypes.byref(d)) == 0


def test_check_rejects_null_workspace(lib):
    assert lib.mamba_mixer_check(None, None) == 1


def _fwd_packed(lib, dims, ptrs=None, ws=None, ws_bytes=0):
    base = 0x10000000
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(
        ["xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias", "seq", "h_in",
         "cs_in", "y", "h", "cs"])}
    if ptrs:
        p.update(ptrs)
    return lib.mamba_mixer_fwd_packed(ctypes.byref(dims), p["xp"], p["z"], p["dt"], p["B"],
                                      p["C"], p["A_log"], p["D"], p["conv_w"], p["conv_b"],
                                      p["dt_bias"], p["seq"], p["h_in"], p["cs_in"], p["y"],
                                      p["h"], p["cs"], ws, ws_bytes, None)


def test_packed_forward_validation(lib):
    d = M.make_dims(2, 64, 128, 16)
    ws = _fake(0x10000000 + 20 * (1 << 36))
    # alignment of the three optional inputs
    assert _fwd_packed(lib, d, {"seq": _fake(0x10000000 + 10 * (1 << 36) + 2)}, ws, 256) == 3
    assert "seq_idx" in M.mamba_last_error()
    assert _fwd_packed(lib, d, {"h_in": _fake(0x10000000 + 11 * (1 << 36) + 8)}, ws, 256) == 3
    assert _fwd_packed(lib, d, {"cs_in": _fake(0x10000000 + 12 * (1 << 36) + 1)}, ws, 256) == 3
    # no in-place update: the final state may not overlap the initial one
    h_in = 0x10000000 + 11 * (1 << 36)
    assert _fwd_packed(lib, d, {"h": _fake(h_in)}, ws, 256) == 1
    assert "overlaps" in M.mamba_last_error()
    cs_in = 0x10000000 + 12 * (1 << 36)
    assert _fwd_packed(lib, d, {"cs": _fake(cs_in)}, ws, 256) == 1
    # an output overlapping seq_idx
    assert _fwd_packed(lib, d, {"y": _fake(0x10000000 + 10 * (1 << 36))}, ws, 256) == 1
    # the workspace rule is the forward's
    assert _fwd_packed(lib, d, ws=None) == 4
    # all optional inputs absent and nothing to do: OK without touching the GPU
    e = M.make_dims(0, 64, 128, 16)
    assert _fwd_packed(lib, e, {k: None for k in ("xp", "z", "dt", "B", "C", "y", "h", "cs",
                                                  "seq", "h_in", "cs_in")}, ws, 256) == 0


def _bwd(lib, dims, ptrs=None, ws=None, ws_bytes=0):
    base = 0x10000000
    names = ["xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias", "dy",
             "dxp", "dz", "ddt", "dB", "dC", "dA_log", "dD", "dconv_w", "dconv_b", "ddt_bias"]
    p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(names)}
    if ptrs:
        p.update(ptrs)
    return lib.mamba_mixer_bwd(ctypes.byref(dims), *[p[k] for k in names], ws, ws_bytes, None)


def test_backward_validation(lib):
    d = M.make_dims(2, 64, 128, 16)
    need = lib.mamba_mixer_bwd_workspace_bytes(ctypes.byref(d))
    assert need == 256 + 2 * 4 * 128 * 16 * 4            # header + four 16-step tile states
    ws = _fake(0x10000000 + 30 * (1 << 36))
    assert _bwd(lib, d, ws=None) == 4                       # workspace required
    assert _bwd(lib, d, ws=ws, ws_bytes=need - 16) == 4
    assert _bwd(lib, d, {"dy": _fake(0x10000000 + 10 * (1 << 36) + 4)}, ws, need) == 3
    assert "dy" in M.mamba_last_error()
    # a gradient output on top of an input or of another output
    assert _bwd(lib, d, {"dxp": _fake(0x10000000 + 0 * (1 << 36))}, ws, need) == 1
    assert _bwd(lib, d, {"dz": _fake(0x10000000 + 11 * (1 << 36))}, ws, need) == 1
    assert _bwd(lib, M.make_dims(2, 64, 128, 12), ws=ws, ws_bytes=need) == 2   # d_state 12
    assert lib.mamba_mixer_bwd_workspace_bytes(ctypes.byref(M.make_dims(2, 64, 128, 12))) == 0


def test_packed_backward_validation(lib):
    d = M.make_dims(2, 64, 128, 16)
    need = lib.mamba_mixer_bwd_workspace_bytes(ctypes.byref(d))
    ws = _fake(0x10000000 + 40 * (1 << 36))
    base = 0x10000000
    names = ["xp", "z", "dt", "B", "C", "A_log", "D", "conv_w", "conv_b", "dt_bias", "seq", "h_in",
             "cs_in", "dy", "dxp", "dz", "ddt", "dB", "dC", "dA_log", "dD", "dconv_w", "dconv_b",
             "ddt_bias", "dh_in", "dcs_in"]

    def call(over):
        p = {k: _fake(base + i * (1 << 36)) for i, k in enumerate(names)}
        p.update(over)
        return lib.mamba_mixer_bwd_packed(ctypes.byref(d), *[p[k] for k in names], ws, need, None)

    assert call({"seq": _fake(base + 10 * (1 << 36) + 2)}) == 3
    assert call({"dh_in": _fake(base + 11 * (1 << 36))}) == 1          # on top of h_in
    assert "overlaps" in M.mamba_last_error()
    assert call({"dcs_in": _fake(base + 24 * (1 << 36) + 2)}) == 3      # fp32 gradient, 4-aligned
