"""Python binding of the Mamba2 scan entry point (include/mamba2_ssd.h) in libmamba_mixer.so.

Argument marshalling only: every step of the computation runs in the library's CUDA
kernel.  The library is the one mixer.load_library() loads; its absence is an error.
"""

from __future__ import annotations

import ctypes
from typing import Optional, Tuple

import torch

from . import mixer as _m

EXPORTS = ("mamba2_ssd_fwd_workspace_bytes", "mamba2_ssd_fwd", "mamba2_ssd_step",
           "mamba2_conv_silu", "mamba2_gated_rmsnorm", "mamba2_ssd_check")


class mamba2_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("nheads", ctypes.c_int64), ("headdim", ctypes.c_int64),
                ("d_state", ctypes.c_int64), ("ngroups", ctypes.c_int64),
                ("io_dtype", ctypes.c_int32), ("reserved", ctypes.c_int32)]


_bound = None


def _lib() -> ctypes.CDLL:
    global _bound
    lib = _m.load_library()
    if _bound is not lib:
        vp = ctypes.c_void_p
        lib.mamba2_ssd_fwd_workspace_bytes.restype = ctypes.c_size_t
        lib.mamba2_ssd_fwd_workspace_bytes.argtypes = [ctypes.POINTER(mamba2_dims)]
        lib.mamba2_ssd_fwd.restype = ctypes.c_int
        lib.mamba2_ssd_fwd.argtypes = [ctypes.POINTER(mamba2_dims)] + [vp] * 13 + [ctypes.c_size_t, vp]
        lib.mamba2_ssd_check.restype = ctypes.c_int
        lib.mamba2_ssd_check.argtypes = [vp]
        lib.mamba2_ssd_step.restype = ctypes.c_int
        lib.mamba2_ssd_step.argtypes = [ctypes.POINTER(mamba2_dims)] + [vp] * 12
        lib.mamba2_conv_silu.restype = ctypes.c_int
        lib.mamba2_conv_silu.argtypes = [ctypes.POINTER(mamba2_dims)] + [vp] * 10
        lib.mamba2_gated_rmsnorm.restype = ctypes.c_int
        lib.mamba2_gated_rmsnorm.argtypes = [ctypes.POINTER(mamba2_dims), vp, vp, vp,
                                             ctypes.c_float, vp, vp]
        _bound = lib
    return lib


def make_dims(batch, seqlen, nheads, headdim, d_state, ngroups, io_dtype=_m.MAMBA_BF16) -> mamba2_dims:
    return mamba2_dims(int(batch), int(seqlen), int(nheads), int(headdim), int(d_state),
                       int(ngroups), int(io_dtype), 0)


def workspace_bytes(dims: mamba2_dims) -> int:
    return int(_lib().mamba2_ssd_fwd_workspace_bytes(ctypes.byref(dims)))


def mamba2_ssd_fwd(x, dt_raw, A_log, B, C, D, dt_bias, *, z=None, seq_idx=None, h_in=None, y=None,
                   h_out=None, want_state: bool = True, workspace=None, stream=None
                   ) -> Tuple[torch.Tensor, Optional[torch.Tensor]]:
    """Mamba2 scan forward.  Shapes: x (and z) [batch, L, nheads, 64] bf16; dt_raw
    [batch, L, nheads] bf16; B, C [batch, L, ngroups, d_state] bf16; A_log, D, dt_bias
    [nheads] fp32; seq_idx [batch, L] int32 or None (documents packed in rows: the state
    resets where the id changes); h_in [batch, nheads, 64, d_state] fp32 or None.  workspace: a uint8
    device tensor of at least workspace_bytes(dims) bytes (allocated when None).  Returns
    (y, h_out) (h_out None when want_state is False)."""
    lib = _lib()
    dev = x.device
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = _m._io_code(x)
    iot = x.dtype
    f32 = torch.float32
    if y is None:
        y = torch.empty_like(x)
    if h_out is None and want_state:
        h_out = torch.empty(Bt, H, P, N, dtype=f32, device=dev)
    dims = make_dims(Bt, L, H, P, N, G, io)
    need = workspace_bytes(dims)
    if workspace is None and need > 0:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    p = _m._ptr
    rc = lib.mamba2_ssd_fwd(
        ctypes.byref(dims), p(x, "x", iot, dev), p(dt_raw, "dt_raw", iot, dev),
        p(A_log, "A_log", f32, dev), p(B, "B", iot, dev), p(C, "C", iot, dev),
        p(D, "D", f32, dev), p(dt_bias, "dt_bias", f32, dev), p(z, "z", iot, dev),
        p(seq_idx, "seq_idx", torch.int32, dev), p(h_in, "h_in", f32, dev), p(y, "y", iot, dev), p(h_out, "h_out", f32, dev),
        p(workspace, "workspace", None, dev), ws_bytes, _m._stream_handle(stream, dev))
    _m._check(rc)
    return y, h_out


def mamba2_ssd_check(stream=None, device=None) -> None:
    """Wait for the stream; raise MambaError(MAMBA_ERR_TIMEOUT) if a mamba2_ssd_fwd since the
    last check gave up on a bounded wait (clears the status)."""
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else torch.device(device)
    _m._check(_lib().mamba2_ssd_check(_m._stream_handle(stream, dev)))


def mamba2_ssd_step(x, dt_raw, A_log, B, C, D, dt_bias, h_in, *, z=None, y=None, h_out=None,
                    stream=None) -> Tuple[torch.Tensor, torch.Tensor]:
    """One decode step: the layouts of mamba2_ssd_fwd with L = 1 (x, z [batch, 1, nheads, 64];
    dt_raw [batch, 1, nheads]; B, C [batch, 1, ngroups, d_state]); h_in [batch, nheads, 64,
    d_state] fp32.  Returns (y, h_out); pass h_out=h_in to update the state in place."""
    lib = _lib()
    dev = x.device
    Bt, L, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    io = _m._io_code(x)
    iot = x.dtype
    f32 = torch.float32
    if y is None:
        y = torch.empty_like(x)
    if h_out is None:
        h_out = torch.empty(Bt, H, P, N, dtype=f32, device=dev)
    dims = make_dims(Bt, L, H, P, N, G, io)
    p = _m._ptr
    rc = lib.mamba2_ssd_step(
        ctypes.byref(dims), p(x, "x", iot, dev), p(dt_raw, "dt_raw", iot, dev),
        p(A_log, "A_log", f32, dev), p(B, "B", iot, dev), p(C, "C", iot, dev),
        p(D, "D", f32, dev), p(dt_bias, "dt_bias", f32, dev), p(z, "z", iot, dev),
        p(h_in, "h_in", f32, dev), p(y, "y", iot, dev), p(h_out, "h_out", f32, dev),
        _m._stream_handle(stream, dev))
    _m._check(rc)
    return y, h_out


def mamba2_conv_silu(xbc, conv_w, conv_b=None, *, nheads, ngroups, d_state, seq_idx=None,
                     conv_state_in=None, want_state: bool = True, stream=None):
    """Causal conv + SiLU over the concatenated x | B | C channels of the Mamba2 layer.
    xbc [batch, L, nheads*64 + 2*ngroups*d_state] bf16; conv_w [channels, 4] fp32; conv_b
    [channels] fp32 or None; seq_idx [batch, L] int32 or None; conv_state_in [batch,
    channels, 3] bf16 or None.  Returns (x [batch, L, nheads, 64], B, C [batch, L, ngroups,
    d_state], conv_state_out [batch, channels, 3] or None), ready for mamba2_ssd_fwd."""
    lib = _lib()
    dev = xbc.device
    Bt, L, Cc = xbc.shape
    iot = xbc.dtype
    H, G, N = int(nheads), int(ngroups), int(d_state)
    x = torch.empty(Bt, L, H, 64, dtype=iot, device=dev)
    B = torch.empty(Bt, L, G, N, dtype=iot, device=dev)
    C = torch.empty(Bt, L, G, N, dtype=iot, device=dev)
    cs_out = torch.empty(Bt, Cc, 3, dtype=iot, device=dev) if want_state else None
    dims = make_dims(Bt, L, H, 64, N, G, _m._io_code(xbc))
    if Cc != H * 64 + 2 * G * N:
        raise ValueError(f"xbc has {Cc} channels, expected {H * 64 + 2 * G * N}")
    p = _m._ptr
    f32 = torch.float32
    rc = lib.mamba2_conv_silu(
        ctypes.byref(dims), p(xbc, "xbc", iot, dev), p(conv_w, "conv_w", f32, dev),
        p(conv_b, "conv_b", f32, dev), p(seq_idx, "seq_idx", torch.int32, dev),
        p(conv_state_in, "conv_state_in", iot, dev), p(x, "x", iot, dev), p(B, "B", iot, dev),
        p(C, "C", iot, dev), p(cs_out, "conv_state_out", iot, dev), _m._stream_handle(stream, dev))
    _m._check(rc)
    return x, B, C, cs_out


def mamba2_gated_rmsnorm(y, z, weight, eps: float = 1e-5, *, ngroups: int = 1, out=None,
                         stream=None):
    """out = y * SiLU(z) normalised to unit RMS over each of ngroups channel groups, times
    weight.  y, z [batch, L, nheads, 64] (or [batch, L, nheads*64]) bf16; weight
    [nheads*64] fp32."""
    lib = _lib()
    dev = y.device
    Bt, L = y.shape[0], y.shape[1]
    D = y.numel() // max(Bt * L, 1) if Bt * L else (y.shape[2] * (y.shape[3] if y.dim() == 4 else 1))
    iot = y.dtype
    if out is None:
        out = torch.empty_like(y)
    dims = make_dims(Bt, L, D // 64, 64, 64, ngroups, _m._io_code(y))
    p = _m._ptr
    rc = lib.mamba2_gated_rmsnorm(
        ctypes.byref(dims), p(y, "y", iot, dev), p(z, "z", iot, dev),
        p(weight, "weight", torch.float32, dev), ctypes.c_float(eps), p(out, "out", iot, dev),
        _m._stream_handle(stream, dev))
    _m._check(rc)
    return out
