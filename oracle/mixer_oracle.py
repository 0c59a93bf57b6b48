"""ctypes wrapper around the plain C oracle (mixer_oracle.c).  TEST INFRASTRUCTURE ONLY.

``build()`` compiles the C file with gcc; ``mixer()`` runs the oracle on numpy arrays.
The arithmetic lives entirely in mixer_oracle_impl.h (a sequential restatement of the
calm-mamba 0.1.4 "Mamba operator" steps 2, 4, 5 and 6); this module only converts
arrays and passes pointers.

Parity status: pinned.  tests/test_oracle_pins.py checks this oracle against closed
forms, library routines (numpy.convolve, numpy.logaddexp, scipy.special.expit,
numpy.cumsum) and an O(L^2) brute-force unrolled sum.
"""

from __future__ import annotations

import ctypes
import os
import subprocess
from typing import Tuple

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "mixer_oracle.c")
_IMPL = os.path.join(_HERE, "mixer_oracle_impl.h")
_BUILD = os.path.join(_HERE, "_build")
_LIB = os.path.join(_BUILD, "liboracle_mixer.so")

GCC_FLAGS = ["-O2", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
             "-Wall", "-Wextra"]

_lib = None


def build(force: bool = False) -> str:
    """Compile the oracle with gcc into oracle/_build/liboracle_mixer.so."""
    os.makedirs(_BUILD, exist_ok=True)
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_IMPL))
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < newest:
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.run(["gcc", *GCC_FLAGS, "-o", tmp, _SRC, "-lm"], check=True)
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(build())
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        for name in ("oracle_mixer_f64", "oracle_mixer_f32"):
            fn = getattr(lib, name)
            fn.restype = ci
            fn.argtypes = [i64] * 5 + [vp] * 16 + [ci]
        lib.oracle_max_threads.restype = ci
        lib.oracle_max_threads.argtypes = []
        _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _arr(a, dt):
    if a is None:
        return None
    return np.ascontiguousarray(a, dtype=dt)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def mixer(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias,
          h_in=None, conv_state_in=None, precision: str = "f64",
          nthreads: int = 1, seq_idx=None) -> Tuple[np.ndarray, np.ndarray, np.ndarray]:
    """Run the oracle.

    Arrays are numeric numpy arrays (already widened from bf16 where that applies) in
    the layouts of mixer_oracle.c.  ``conv_b``, ``h_in`` and ``conv_state_in`` may be
    None (zero bias; zero initial state).  ``seq_idx`` ([Bt, L] integers, optional) marks
    packed documents: the conv and SSM states reset wherever it changes along t.  Returns (y [Bt,L,Di], h_out [Bt,Di,N],
    conv_state_out [Bt,Di,K-1]) in the requested precision ("f64" or "f32").
    """
    dt = {"f64": np.float64, "f32": np.float32}[precision]
    fn = getattr(_load(), f"oracle_mixer_{precision}")
    xp, z, dt_raw = _arr(xp, dt), _arr(z, dt), _arr(dt_raw, dt)
    B, C = _arr(B, dt), _arr(C, dt)
    A_log, D, conv_w = _arr(A_log, dt), _arr(D, dt), _arr(conv_w, dt)
    conv_b, dt_bias = _arr(conv_b, dt), _arr(dt_bias, dt)
    h_in, conv_state_in = _arr(h_in, dt), _arr(conv_state_in, dt)
    seq_idx = _arr(seq_idx, np.int32)
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    assert z.shape == xp.shape and dt_raw.shape == xp.shape
    assert B.shape == (Bt, L, N) and C.shape == (Bt, L, N)
    assert A_log.shape == (Di, N) and D.shape == (Di,) and dt_bias.shape == (Di,)
    assert conv_b is None or conv_b.shape == (Di,)
    assert h_in is None or h_in.shape == (Bt, Di, N)
    assert conv_state_in is None or conv_state_in.shape == (Bt, Di, K - 1)
    assert seq_idx is None or seq_idx.shape == (Bt, L)
    y = np.empty((Bt, L, Di), dtype=dt)
    h_out = np.empty((Bt, Di, N), dtype=dt)
    cs_out = np.empty((Bt, Di, K - 1), dtype=dt)
    rc = fn(Bt, L, Di, N, K, _ptr(xp), _ptr(z), _ptr(dt_raw), _ptr(B), _ptr(C), _ptr(A_log),
            _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(dt_bias), _ptr(seq_idx), _ptr(h_in),
            _ptr(conv_state_in), _ptr(y), _ptr(h_out), _ptr(cs_out), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle failed with code {rc}")
    return y, h_out, cs_out


def mixer_channels(inp: dict, batch_idx, chan_idx, precision: str = "f64",
                   nthreads: int = 1, widen=None):
    """Oracle over a subset of channels of one workload's inputs.

    Every channel (b, d) of the mixer is independent given B[b], C[b] and the
    parameters of d, so the selected channels form a smaller problem: batch rows
    ``batch_idx`` and channels ``chan_idx`` (all pairs).  ``widen`` maps a stored
    activation to float64 (bf16 bit patterns are widened exactly).  Returns the outputs
    of the sub-problem with shapes [len(batch_idx), L, len(chan_idx)] etc.
    """
    bi = np.asarray(batch_idx)
    di = np.asarray(chan_idx)
    w = widen or (lambda a: np.asarray(a, dtype=np.float64))
    sub = {
        "xp": w(inp["xp"][bi][:, :, di]),
        "z": w(inp["z"][bi][:, :, di]),
        "dt_raw": w(inp["dt_raw"][bi][:, :, di]),
        "B": w(inp["B"][bi]),
        "C": w(inp["C"][bi]),
        "A_log": inp["A_log"][di],
        "D": inp["D"][di],
        "conv_w": inp["conv_w"][di],
        "conv_b": None if inp.get("conv_b") is None else inp["conv_b"][di],
        "dt_bias": inp["dt_bias"][di],
    }
    h_in = inp.get("h")
    cs_in = inp.get("conv_state")
    if h_in is not None:
        h_in = h_in[bi][:, di]
    if cs_in is not None:
        cs_in = w(cs_in[bi][:, di])
    seq = inp.get("seq_idx")
    if seq is not None:
        seq = seq[bi]
    return mixer(sub["xp"], sub["z"], sub["dt_raw"], sub["B"], sub["C"], sub["A_log"],
                 sub["D"], sub["conv_w"], sub["conv_b"], sub["dt_bias"], h_in, cs_in,
                 precision=precision, nthreads=nthreads, seq_idx=seq)


def mixer_dtproj(xp, z, dt_low, W_dt, B, C, A_log, D, conv_w, conv_b, dt_bias, nthreads: int = 1):
    """The forward with the dt projection fused (calm-mamba 0.1.4, "Mamba operator", step 4:
    dt = dt_proj(dt_low)): dt_raw = dt_low W_dt^T, a library matmul in fp64 with no rounding
    between the two steps, then the mixer oracle above.  dt_low [Bt, L, R], W_dt [Di, R]."""
    dt_raw = np.matmul(np.asarray(dt_low, dtype=np.float64), np.asarray(W_dt, dtype=np.float64).T)
    return mixer(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, nthreads=nthreads)


def mixer_dtproj_channels(inp: dict, batch_idx, chan_idx, nthreads: int = 1, widen=None):
    """mixer_dtproj over a subset of channels (as mixer_channels): the projection is formed
    for the selected batch rows and channels only, dt_raw[b, :, d] = dt_low[b] W_dt[d]^T."""
    w = widen or (lambda a: np.asarray(a, dtype=np.float64))
    bi = np.asarray(batch_idx)
    di = np.asarray(chan_idx)
    dt_raw = np.matmul(w(inp["dt_low"][bi]), w(inp["W_dt"][di]).T)
    cb = inp.get("conv_b")
    return mixer(w(inp["xp"][bi][:, :, di]), w(inp["z"][bi][:, :, di]), dt_raw, w(inp["B"][bi]),
                 w(inp["C"][bi]), inp["A_log"][di], inp["D"][di], inp["conv_w"][di],
                 None if cb is None else cb[di], inp["dt_bias"][di], nthreads=nthreads)


BWD_NAMES = ("dxp", "dz", "ddt_raw", "dB", "dC", "dA_log", "dD", "dconv_w", "dconv_b", "ddt_bias")


def mixer_bwd(xp, z, dt_raw, B, C, A_log, D, conv_w, conv_b, dt_bias, dy, nthreads: int = 1,
              seq_idx=None, h_in=None, conv_state_in=None):
    """Gradients of sum(dy * y) with respect to every forward input (fp64 oracle).  Returns
    a dict keyed by BWD_NAMES (dconv_b None without conv_b), plus "dh_in" and
    "dconv_state_in" (None unless the forward started from that cached state)."""
    lib = _load()
    fn = lib.oracle_mixer_bwd_f64
    if getattr(fn, "_typed", None) is None:
        i64, vp, ci = ctypes.c_int64, ctypes.c_void_p, ctypes.c_int
        fn.restype = ci
        fn.argtypes = [i64] * 5 + [vp] * 26 + [ci]
        fn._typed = True
    f = np.float64
    xp, z, dt_raw, B, C = (_arr(a, f) for a in (xp, z, dt_raw, B, C))
    A_log, D, conv_w, dt_bias, dy = (_arr(a, f) for a in (A_log, D, conv_w, dt_bias, dy))
    conv_b = _arr(conv_b, f)
    seq_idx = _arr(seq_idx, np.int32)
    h_in, conv_state_in = _arr(h_in, f), _arr(conv_state_in, f)
    Bt, L, Di = xp.shape
    N = A_log.shape[1]
    K = conv_w.shape[1]
    assert dy.shape == xp.shape
    out = {
        "dxp": np.empty((Bt, L, Di)), "dz": np.empty((Bt, L, Di)), "ddt_raw": np.empty((Bt, L, Di)),
        "dB": np.empty((Bt, L, N)), "dC": np.empty((Bt, L, N)), "dA_log": np.empty((Di, N)),
        "dD": np.empty(Di), "dconv_w": np.empty((Di, K)),
        "dconv_b": None if conv_b is None else np.empty(Di), "ddt_bias": np.empty(Di),
        "dh_in": None if h_in is None else np.empty((Bt, Di, N)),
        "dconv_state_in": None if conv_state_in is None else np.empty((Bt, Di, K - 1)),
    }
    rc = fn(Bt, L, Di, N, K, _ptr(xp), _ptr(z), _ptr(dt_raw), _ptr(B), _ptr(C), _ptr(A_log),
            _ptr(D), _ptr(conv_w), _ptr(conv_b), _ptr(dt_bias), _ptr(seq_idx), _ptr(h_in),
            _ptr(conv_state_in), _ptr(dy), *[_ptr(out[k]) for k in BWD_NAMES],
            _ptr(out["dh_in"]), _ptr(out["dconv_state_in"]), int(nthreads))
    if rc != 0:
        raise RuntimeError(f"backward oracle failed with code {rc}")
    return out
