"""Python binding of libmamba_mixer.so (include/mamba_mixer.h), by ctypes.

Argument marshalling only: torch tensors are checked for device, dtype and contiguity,
their data pointers and the current CUDA stream are passed to the C entry points of the
same names, and a non-OK status becomes a ``MambaError``.  Every step of the mixer runs
in the library's CUDA kernels; there is no other implementation behind these calls.
Missing outputs (and the forward's workspace) are allocated with ``torch.empty``.
"""

from __future__ import annotations

import ctypes
import os
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libmamba_mixer.so")

MAMBA_F32 = 0
MAMBA_BF16 = 1
STATUS = {0: "MAMBA_OK", 1: "MAMBA_ERR_INVALID_ARGUMENT", 2: "MAMBA_ERR_UNSUPPORTED",
          3: "MAMBA_ERR_ALIGNMENT", 4: "MAMBA_ERR_WORKSPACE", 5: "MAMBA_ERR_CUDA",
          6: "MAMBA_ERR_TIMEOUT"}
EXPORTS = ("mamba_mixer_fwd_workspace_bytes", "mamba_mixer_fwd_launches", "mamba_mixer_fwd",
           "mamba_mixer_fwd_packed", "mamba_mixer_bwd_workspace_bytes", "mamba_mixer_bwd",
           "mamba_mixer_bwd_packed",
           "mamba_mixer_step", "mamba_mixer_step_check", "mamba_mixer_check",
           "mamba_mixer_set_fault_injection", "mamba_mixer_ckpt_bytes", "mamba_mixer_fwd_ckpt",
           "mamba_mixer_bwd_ckpt",
           "mamba_mixer_fwd_plan", "mamba_mixer_fwd_dtproj",
           "mamba_mixer_fwd_noalloc",
           "mamba_mixer_noalloc_check", "mamba_last_error", "mamba_version")


class MambaError(RuntimeError):
    def __init__(self, code: int, msg: str):
        super().__init__(f"{STATUS.get(code, code)}: {msg}")
        self.code = code


class mamba_dims(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int64), ("seqlen", ctypes.c_int64),
                ("d_inner", ctypes.c_int64), ("d_state", ctypes.c_int64),
                ("d_conv", ctypes.c_int64), ("io_dtype", ctypes.c_int32),
                ("reserved", ctypes.c_int32)]


_lib = None


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load the CUDA library; raises if it is missing (build it first)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(
            f"{path} is missing: build it with `python -m selective_state_space_silu_b200.build` "
            "(there is no fallback implementation)")
    lib = ctypes.CDLL(path)
    vp, i, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
    P = ctypes.POINTER(mamba_dims)
    lib.mamba_mixer_fwd_workspace_bytes.restype = sz
    lib.mamba_mixer_fwd_workspace_bytes.argtypes = [P]
    lib.mamba_mixer_fwd_launches.restype = i
    lib.mamba_mixer_fwd_launches.argtypes = [P]
    lib.mamba_mixer_check.restype = i
    lib.mamba_mixer_check.argtypes = [vp, vp]
    lib.mamba_mixer_set_fault_injection.restype = None
    lib.mamba_mixer_set_fault_injection.argtypes = [i]
    lib.mamba_mixer_ckpt_bytes.restype = sz
    lib.mamba_mixer_ckpt_bytes.argtypes = [P]
    lib.mamba_mixer_fwd_ckpt.restype = i
    lib.mamba_mixer_fwd_ckpt.argtypes = [P] + [vp] * 14 + [vp, sz, vp]
    lib.mamba_mixer_bwd_ckpt.restype = i
    lib.mamba_mixer_bwd_ckpt.argtypes = [P] + [vp] * 12 + [vp] * 10 + [vp, sz, vp]
    lib.mamba_mixer_fwd.restype = i
    lib.mamba_mixer_fwd.argtypes = [P] + [vp] * 13 + [vp, sz, vp]
    lib.mamba_mixer_fwd_packed.restype = i
    lib.mamba_mixer_fwd_packed.argtypes = [P] + [vp] * 16 + [vp, sz, vp]
    lib.mamba_mixer_bwd_workspace_bytes.restype = sz
    lib.mamba_mixer_bwd_workspace_bytes.argtypes = [P]
    lib.mamba_mixer_bwd.restype = i
    lib.mamba_mixer_bwd.argtypes = [P] + [vp] * 21 + [vp, sz, vp]
    lib.mamba_mixer_bwd_packed.restype = i
    lib.mamba_mixer_bwd_packed.argtypes = [P] + [vp] * 26 + [vp, sz, vp]
    lib.mamba_mixer_step.restype = i
    lib.mamba_mixer_step.argtypes = [P] + [vp] * 15 + [vp]
    lib.mamba_last_error.restype = ctypes.c_char_p
    lib.mamba_last_error.argtypes = []
    lib.mamba_version.restype = ctypes.c_char_p
    lib.mamba_version.argtypes = []
    _lib = lib
    return lib


def mamba_version() -> str:
    return load_library().mamba_version().decode()


def mamba_last_error() -> str:
    return load_library().mamba_last_error().decode()


def make_dims(batch, seqlen, d_inner, d_state, d_conv=4, io_dtype=MAMBA_BF16) -> mamba_dims:
    return mamba_dims(int(batch), int(seqlen), int(d_inner), int(d_state), int(d_conv),
                      int(io_dtype), 0)


def _io_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return MAMBA_F32
    if t.dtype == torch.bfloat16:
        return MAMBA_BF16
    raise TypeError(f"activations must be float32 or bfloat16, got {t.dtype}")


def _ptr(t: Optional[torch.Tensor], name: str, dtype=None, device=None):
    if t is None:
        return None
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} has dtype {t.dtype}, expected {dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t.data_ptr() if t.numel() > 0 else None


def _stream_handle(stream, device) -> Optional[int]:
    s = stream if stream is not None else torch.cuda.current_stream(device)
    return s.cuda_stream


def _check(rc: int):
    if rc != 0:
        raise MambaError(rc, mamba_last_error())


def mamba_mixer_fwd_workspace_bytes(dims: mamba_dims) -> int:
    return int(load_library().mamba_mixer_fwd_workspace_bytes(ctypes.byref(dims)))


def mamba_mixer_bwd_workspace_bytes(dims: mamba_dims) -> int:
    return int(load_library().mamba_mixer_bwd_workspace_bytes(ctypes.byref(dims)))


def new_workspace(dims: mamba_dims, device) -> torch.Tensor:
    """A zeroed workspace of the size mamba_mixer_fwd needs for ``dims``."""
    need = mamba_mixer_fwd_workspace_bytes(dims)
    if need == 0:
        raise MambaError(2, "unsupported dims: " + mamba_last_error())
    return torch.zeros(need, dtype=torch.uint8, device=device)


def mamba_mixer_check(workspace: torch.Tensor, stream=None) -> None:
    """Wait for the stream; raise MambaError(MAMBA_ERR_TIMEOUT) if a forward that used
    ``workspace`` gave up on a bounded wait since the last check (clears the status)."""
    rc = load_library().mamba_mixer_check(workspace.data_ptr(),
                                          _stream_handle(stream, workspace.device))
    _check(rc)


def mamba_mixer_set_fault_injection(tile: int) -> None:
    """Test hook: tile >= 0 makes one CTA of every following forward skip the copies of
    its time tile ``tile`` so that its bounded waits run out (MAMBA_ERR_TIMEOUT, no GPU
    fault); -1 turns it off."""
    load_library().mamba_mixer_set_fault_injection(int(tile))


def mamba_mixer_fwd(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, *,
                    y=None, h_out=None, conv_state_out=None, workspace=None,
                    stream=None, want_states: bool = True, h_ckpt=None
                    ) -> Tuple[torch.Tensor, Optional[torch.Tensor], Optional[torch.Tensor]]:
    """Fused forward (conv + SiLU, softplus, selective scan, gate) from a zero state.

    Shapes: xp, z, dt_raw [batch, L, d_inner]; B, C [batch, L, d_state]; A_log
    [d_inner, d_state]; D, dt_bias, conv_b [d_inner]; conv_w [d_inner, 4].  Returns
    (y, h_out, conv_state_out).  With ``h_ckpt`` (fp32 [batch, ceil(L/16), d_inner,
    d_state], see ``new_ckpt``) it also writes the state before every 16-step tile
    (mamba_mixer_fwd_ckpt), which ``mamba_mixer_bwd(..., h_ckpt=)`` then reads.
    """
    lib = load_library()
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    dims = make_dims(Bt, L, Di, N, K, io)
    if y is None:
        y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
    if want_states and h_out is None:
        h_out = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    if want_states and conv_state_out is None:
        conv_state_out = torch.empty((Bt, Di, K - 1), dtype=iot, device=dev)
    if workspace is None:
        workspace = new_workspace(dims, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    f32 = torch.float32
    args = [ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
            _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
            _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev),
            _ptr(conv_w, "conv_w", f32, dev), _ptr(conv_b, "conv_b", f32, dev),
            _ptr(dt_bias, "dt_bias", f32, dev), _ptr(y, "y", iot, dev),
            _ptr(h_out, "h_out", f32, dev), _ptr(conv_state_out, "conv_state_out", iot, dev)]
    tail = [_ptr(workspace, "workspace", None, dev), ws_bytes, _stream_handle(stream, dev)]
    if h_ckpt is None:
        rc = lib.mamba_mixer_fwd(*args, *tail)
    else:
        rc = lib.mamba_mixer_fwd_ckpt(*args, _ptr(h_ckpt, "h_ckpt", f32, dev), *tail)
    _check(rc)
    return y, h_out, conv_state_out


def new_ckpt(dims: mamba_dims, device) -> torch.Tensor:
    """The state checkpoints of mamba_mixer_fwd_ckpt for ``dims``: fp32 [batch,
    ceil(L/16), d_inner, d_state]."""
    t16 = (dims.seqlen + 15) // 16
    return torch.empty((dims.batch, t16, dims.d_inner, dims.d_state), dtype=torch.float32,
                       device=device)


def mamba_mixer_fwd_packed(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, *,
                           seq_idx=None, h_in=None, conv_state_in=None, y=None, h_out=None,
                           conv_state_out=None, workspace=None, stream=None
                           ) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """Fused forward over packed documents and/or from a cached state.

    As mamba_mixer_fwd, plus optional seq_idx [batch, L] int32 (the states reset wherever
    the id changes along t), h_in [batch, d_inner, d_state] fp32 and conv_state_in
    [batch, d_inner, 3] (the state before token 0).  Returns (y, h_out, conv_state_out).
    """
    lib = load_library()
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    dims = make_dims(Bt, L, Di, N, K, io)
    if y is None:
        y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
    if h_out is None:
        h_out = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    if conv_state_out is None:
        conv_state_out = torch.empty((Bt, Di, K - 1), dtype=iot, device=dev)
    if workspace is None:
        workspace = new_workspace(dims, dev)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    f32 = torch.float32
    rc = lib.mamba_mixer_fwd_packed(
        ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
        _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
        _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev), _ptr(conv_w, "conv_w", f32, dev),
        _ptr(conv_b, "conv_b", f32, dev), _ptr(dt_bias, "dt_bias", f32, dev),
        _ptr(seq_idx, "seq_idx", torch.int32, dev), _ptr(h_in, "h_in", f32, dev),
        _ptr(conv_state_in, "conv_state_in", iot, dev),
        _ptr(y, "y", iot, dev), _ptr(h_out, "h_out", f32, dev),
        _ptr(conv_state_out, "conv_state_out", iot, dev),
        _ptr(workspace, "workspace", None, dev), ws_bytes, _stream_handle(stream, dev))
    _check(rc)
    return y, h_out, conv_state_out


BWD_OUTPUTS = ("dxp", "dz", "ddt_raw", "dB", "dC", "dA_log", "dD", "dconv_w", "dconv_b",
               "ddt_bias")


def mamba_mixer_bwd(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, dy, *,
                    workspace=None, stream=None, h_ckpt=None) -> dict:
    """Gradients of sum(dy * y) for mamba_mixer_fwd, all fp32; returns a dict keyed by
    BWD_OUTPUTS (dconv_b is None when conv_b is None).  With ``h_ckpt`` (written by
    mamba_mixer_fwd(..., h_ckpt=) on the same inputs) the backward reads the tile states
    instead of recomputing them (mamba_mixer_bwd_ckpt)."""
    lib = load_library()
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    dims = make_dims(Bt, L, Di, N, K, io)
    f32 = torch.float32
    e = lambda *shape: torch.empty(shape, dtype=f32, device=dev)
    g = {"dxp": e(Bt, L, Di), "dz": e(Bt, L, Di), "ddt_raw": e(Bt, L, Di), "dB": e(Bt, L, N),
         "dC": e(Bt, L, N), "dA_log": e(Di, N), "dD": e(Di), "dconv_w": e(Di, K),
         "dconv_b": None if conv_b is None else e(Di), "ddt_bias": e(Di)}
    need = int(lib.mamba_mixer_bwd_workspace_bytes(ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    ins = [ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
           _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
           _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev),
           _ptr(conv_w, "conv_w", f32, dev), _ptr(conv_b, "conv_b", f32, dev),
           _ptr(dt_bias, "dt_bias", f32, dev)]
    rest = [_ptr(dy, "dy", iot, dev), *[_ptr(g[k], k, f32, dev) for k in BWD_OUTPUTS],
            _ptr(workspace, "workspace", None, dev), ws_bytes, _stream_handle(stream, dev)]
    if h_ckpt is None:
        rc = lib.mamba_mixer_bwd(*ins, *rest)
    else:
        rc = lib.mamba_mixer_bwd_ckpt(*ins, _ptr(h_ckpt, "h_ckpt", f32, dev), *rest)
    _check(rc)
    return g


def mamba_mixer_bwd_packed(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, dy, *,
                           seq_idx=None, h_in=None, conv_state_in=None, want_state_grads=True,
                           workspace=None, stream=None) -> dict:
    """Gradients of sum(dy * y) for mamba_mixer_fwd_packed (documents and/or a cached
    start), all fp32: the keys of BWD_OUTPUTS plus "dh_in" and "dconv_state_in" (None when
    want_state_grads is False)."""
    lib = load_library()
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    dims = make_dims(Bt, L, Di, N, K, io)
    f32 = torch.float32
    e = lambda *shape: torch.empty(shape, dtype=f32, device=dev)
    g = {"dxp": e(Bt, L, Di), "dz": e(Bt, L, Di), "ddt_raw": e(Bt, L, Di), "dB": e(Bt, L, N),
         "dC": e(Bt, L, N), "dA_log": e(Di, N), "dD": e(Di), "dconv_w": e(Di, K),
         "dconv_b": None if conv_b is None else e(Di), "ddt_bias": e(Di),
         "dh_in": e(Bt, Di, N) if want_state_grads else None,
         "dconv_state_in": e(Bt, Di, K - 1) if want_state_grads else None}
    need = int(lib.mamba_mixer_bwd_workspace_bytes(ctypes.byref(dims)))
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    ws_bytes = workspace.numel() * workspace.element_size()
    rc = lib.mamba_mixer_bwd_packed(
        ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
        _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
        _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev), _ptr(conv_w, "conv_w", f32, dev),
        _ptr(conv_b, "conv_b", f32, dev), _ptr(dt_bias, "dt_bias", f32, dev),
        _ptr(seq_idx, "seq_idx", torch.int32, dev), _ptr(h_in, "h_in", f32, dev),
        _ptr(conv_state_in, "conv_state_in", iot, dev), _ptr(dy, "dy", iot, dev),
        *[_ptr(g[k], k, f32, dev) for k in BWD_OUTPUTS],
        _ptr(g["dh_in"], "dh_in", f32, dev), _ptr(g["dconv_state_in"], "dconv_state_in", f32, dev),
        _ptr(workspace, "workspace", None, dev), ws_bytes, _stream_handle(stream, dev))
    _check(rc)
    return g


def mamba_mixer_step(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, h_in,
                     conv_state_in, *, y=None, h_out=None, conv_state_out=None,
                     stream=None) -> Tuple[torch.Tensor, torch.Tensor, torch.Tensor]:
    """One decode step on a cached state; functional unless outputs alias the inputs.

    Shapes: xp, z, dt_raw [batch, 1, d_inner] (or [batch, d_inner]); B, C [batch, 1,
    d_state] (or [batch, d_state]); h_in [batch, d_inner, d_state] fp32; conv_state_in
    [batch, d_inner, 3].  Returns (y, h_out, conv_state_out); pass h_out=h_in and
    conv_state_out=conv_state_in for an in-place update.
    """
    lib = load_library()
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, Di, N = h_in.shape
    K = conv_w.shape[1]
    dims = make_dims(Bt, 1, Di, N, K, io)
    if y is None:
        y = torch.empty(xp.shape, dtype=iot, device=dev)
    if h_out is None:
        h_out = torch.empty_like(h_in)
    if conv_state_out is None:
        conv_state_out = torch.empty_like(conv_state_in)
    f32 = torch.float32
    rc = lib.mamba_mixer_step(
        ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
        _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
        _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev), _ptr(conv_w, "conv_w", f32, dev),
        _ptr(conv_b, "conv_b", f32, dev), _ptr(dt_bias, "dt_bias", f32, dev),
        _ptr(h_in, "h_in", f32, dev), _ptr(conv_state_in, "conv_state_in", iot, dev),
        _ptr(y, "y", iot, dev), _ptr(h_out, "h_out", f32, dev),
        _ptr(conv_state_out, "conv_state_out", iot, dev), _stream_handle(stream, dev))
    _check(rc)
    return y, h_out, conv_state_out


def mamba_mixer_fwd_dtproj(xp, z, dt_low, W_dt, B, C, A_log, D, conv_w, conv_b, dt_bias, *,
                           y=None, h_out=None, conv_state_out=None, workspace=None,
                           stream=None, want_states: bool = True):
    """The fused forward with the dt projection folded in: dt_raw = dt_low W_dt^T is formed
    per tile on the tensor cores.  dt_low [batch, L, dt_rank] and W_dt [d_inner, dt_rank] are
    bf16; every other argument and the results are those of ``mamba_mixer_fwd`` (bf16 I/O)."""
    lib = load_library()
    lib.mamba_mixer_fwd_dtproj.restype = ctypes.c_int
    lib.mamba_mixer_fwd_dtproj.argtypes = ([ctypes.POINTER(mamba_dims), ctypes.c_int64] +
                                           [ctypes.c_void_p] * 15 + [ctypes.c_size_t, ctypes.c_void_p])
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    R = dt_low.shape[2]
    if tuple(W_dt.shape) != (Di, R) or tuple(dt_low.shape[:2]) != (Bt, L):
        raise MambaError(1, "dt_low must be [batch, L, dt_rank] and W_dt [d_inner, dt_rank]")
    dims = make_dims(Bt, L, Di, N, K, io)
    if y is None:
        y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
    if want_states and h_out is None:
        h_out = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    if want_states and conv_state_out is None:
        conv_state_out = torch.empty((Bt, Di, K - 1), dtype=iot, device=dev)
    if workspace is None:
        workspace = new_workspace(dims, dev)
    f32 = torch.float32
    rc = lib.mamba_mixer_fwd_dtproj(
        ctypes.byref(dims), R, _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
        _ptr(dt_low, "dt_low", torch.bfloat16, dev), _ptr(W_dt, "W_dt", torch.bfloat16, dev),
        _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
        _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev), _ptr(conv_w, "conv_w", f32, dev),
        _ptr(conv_b, "conv_b", f32, dev), _ptr(dt_bias, "dt_bias", f32, dev),
        _ptr(y, "y", iot, dev), _ptr(h_out, "h_out", f32, dev),
        _ptr(conv_state_out, "conv_state_out", iot, dev),
        workspace.data_ptr(), workspace.numel() * workspace.element_size(),
        _stream_handle(stream, dev))
    _check(rc)
    return y, h_out, conv_state_out


def mamba_mixer_fwd_plan(dims: mamba_dims) -> dict:
    """How the forward splits ``dims``: nchunks, chunk_len, time_groups, chained."""
    lib = load_library()
    lib.mamba_mixer_fwd_plan.restype = ctypes.c_int
    lib.mamba_mixer_fwd_plan.argtypes = [ctypes.POINTER(mamba_dims), ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_int64), ctypes.POINTER(ctypes.c_int),
                                         ctypes.POINTER(ctypes.c_int)]
    n, g, ch = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    ln = ctypes.c_int64()
    _check(lib.mamba_mixer_fwd_plan(ctypes.byref(dims), ctypes.byref(n), ctypes.byref(ln),
                                    ctypes.byref(g), ctypes.byref(ch)))
    return {"nchunks": n.value, "chunk_len": ln.value, "time_groups": g.value,
            "chained": bool(ch.value)}


def mamba_mixer_fwd_launches(dims: mamba_dims) -> int:
    """Kernel launches one mamba_mixer_fwd call with ``dims`` makes."""
    return int(load_library().mamba_mixer_fwd_launches(ctypes.byref(dims)))


def mamba_mixer_fwd_noalloc(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, *,
                            y=None, h_out=None, conv_state_out=None, stream=None,
                            want_states: bool = True):
    """The fused forward without a workspace, for callers that cannot allocate device
    memory: the library uses its own fixed 2 MiB scratch array per device instead.

    Same arguments and results as ``mamba_mixer_fwd`` minus ``workspace``.  Calls on one
    device share that scratch, so calls that overlap on the GPU race; sizes needing more
    scratch than 2 MiB raise MambaError(MAMBA_ERR_WORKSPACE).  (This binding still creates
    output tensors when they are not given; pass them in to allocate nothing.)
    """
    lib = load_library()
    lib.mamba_mixer_fwd_noalloc.restype = ctypes.c_int
    lib.mamba_mixer_fwd_noalloc.argtypes = [ctypes.POINTER(mamba_dims)] + [ctypes.c_void_p] * 14
    dev = xp.device
    io = _io_code(xp)
    iot = xp.dtype
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    dims = make_dims(Bt, L, Di, N, K, io)
    if y is None:
        y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
    if want_states and h_out is None:
        h_out = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    if want_states and conv_state_out is None:
        conv_state_out = torch.empty((Bt, Di, K - 1), dtype=iot, device=dev)
    f32 = torch.float32
    rc = lib.mamba_mixer_fwd_noalloc(
        ctypes.byref(dims), _ptr(xp, "xp", iot, dev), _ptr(z, "z", iot, dev),
        _ptr(dt_raw, "dt_raw", iot, dev), _ptr(B, "B", iot, dev), _ptr(C, "C", iot, dev),
        _ptr(A_log, "A_log", f32, dev), _ptr(D, "D", f32, dev), _ptr(conv_w, "conv_w", f32, dev),
        _ptr(conv_b, "conv_b", f32, dev), _ptr(dt_bias, "dt_bias", f32, dev),
        _ptr(y, "y", iot, dev), _ptr(h_out, "h_out", f32, dev),
        _ptr(conv_state_out, "conv_state_out", iot, dev), _stream_handle(stream, dev))
    _check(rc)
    return y, h_out, conv_state_out


def mamba_mixer_step_check(stream=None, device=None) -> None:
    """Wait for the stream; raise MambaError(MAMBA_ERR_TIMEOUT) if a decode step in the
    current context gave up on a bounded wait since the last check (clears the status)."""
    lib = load_library()
    lib.mamba_mixer_step_check.restype = ctypes.c_int
    lib.mamba_mixer_step_check.argtypes = [ctypes.c_void_p]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check(lib.mamba_mixer_step_check(_stream_handle(stream, dev)))


def mamba_mixer_noalloc_check(stream=None, device=None) -> None:
    """Wait for the stream; raise MambaError(MAMBA_ERR_TIMEOUT) if a no-alloc forward in
    the current context gave up on a bounded wait since the last check (clears the status).
    Allocates nothing."""
    lib = load_library()
    lib.mamba_mixer_noalloc_check.restype = ctypes.c_int
    lib.mamba_mixer_noalloc_check.argtypes = [ctypes.c_void_p]
    dev = torch.device("cuda", torch.cuda.current_device()) if device is None else device
    _check(lib.mamba_mixer_noalloc_check(_stream_handle(stream, dev)))


class MambaMixerFunction(torch.autograd.Function):
    """The fused forward as a differentiable op: forward = mamba_mixer_fwd (from a zero
    state), backward = mamba_mixer_bwd; gradients come back in each input's dtype.  With
    checkpoint_states the forward also keeps the state before every 16-step tile (fp32,
    4 * d_state bytes per token and channel / 16) and the backward reads them instead of
    recomputing them."""

    @staticmethod
    def forward(ctx, xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, checkpoint_states):
        xp, z, dt_raw, B, C = (t.contiguous() for t in (xp, z, dt_raw, B, C))
        ck = None
        if checkpoint_states:
            Bt, L, Di = xp.shape
            ck = new_ckpt(make_dims(Bt, L, Di, A_log.shape[1], conv_w.shape[1], _io_code(xp)),
                          xp.device)
        y, _, _ = mamba_mixer_fwd(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias,
                                  want_states=False, h_ckpt=ck)
        ctx.save_for_backward(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, ck)
        return y

    @staticmethod
    def backward(ctx, dy):
        xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, ck = ctx.saved_tensors
        g = mamba_mixer_bwd(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias,
                            dy.to(xp.dtype).contiguous(), h_ckpt=ck)
        as_ = lambda k, ref: None if g[k] is None else g[k].to(ref.dtype)
        return (as_("dxp", xp), as_("dz", z), as_("ddt_raw", dt_raw), as_("dB", B), as_("dC", C),
                as_("dA_log", A_log), as_("dD", D), as_("dconv_w", conv_w),
                None if conv_b is None else as_("dconv_b", conv_b), as_("ddt_bias", dt_bias),
                None)


def mamba_mixer(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, *,
                checkpoint_states: bool = False):
    """y = the fused mixer forward, differentiable with respect to every input."""
    return MambaMixerFunction.apply(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias,
                                    checkpoint_states)
