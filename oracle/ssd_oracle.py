"""Plain fp64 CPU oracle for the Mamba2 selective scan (the SSD layer).  TEST INFRASTRUCTURE
ONLY: tests, the smoke check and the benchmark's CPU baseline call it; nothing on the
product path does.

What it computes (niverel-mamba 0.1.0, sections "The weight contract", "seq_idx strict
reset" and "Measured tolerances"): the Mamba recurrence of the calm-mamba 0.1.4 "Mamba
operator" with the Mamba2 parametrisation -- one scalar A, one Delta and one D per head,
shared by the head's ``P`` channels (headdim), and one B/C pair per group of heads
(ngroups).  For every batch row b, head h (group g = h // (H / G)), channel p, state n:

    Delta_t   = softplus(dt_raw[b,t,h] + dt_bias[h])           softplus(v) = log(1 + e^v)
    A         = -exp(A_log[h])
    h[p, n]  <- exp(Delta_t * A) * h[p, n] + Delta_t * x[b,t,h,p] * B[b,t,g,n]
    y[b,t,h,p] = sum_n C[b,t,g,n] * h[p, n] + D[h] * x[b,t,h,p]
    out       = y * SiLU(z[b,t,h,p])          (only when z is given; SiLU(v) = v / (1 + e^-v))

x is the activation after the causal conv and SiLU (the layer's conv runs before the scan).
The state starts from h_in (zero when absent) and is zeroed before every step t > 0 whose
seq_idx differs from step t - 1's.  The final state is returned as h_out [Bt, H, P, N].

The loop runs over time in order, one step per iteration, vectorised over (b, h, p, n)
only: no chunking, no reordering.  The chunked (quadratic-within-a-chunk) evaluation is
what the CUDA path does; tests/test_oracle_ssd.py checks this oracle against that form
written out independently, an O(L^2) unrolled sum, closed forms and numpy.cumsum.

The same module holds the layer's two neighbours of the scan: conv_silu (the causal
depthwise conv + SiLU over the concatenated x, B, C channels) and gated_rmsnorm (the norm
of y * SiLU(z)).

Parity status: pinned (tests/test_oracle_ssd.py).
"""

from __future__ import annotations

from typing import Optional, Tuple

import numpy as np


def as_f64(a) -> np.ndarray:
    """An activation as fp64: bf16 bit patterns (uint16) are widened exactly."""
    a = np.asarray(a)
    if a.dtype == np.uint16:
        return (a.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    return a.astype(np.float64)


def _softplus(v: np.ndarray) -> np.ndarray:
    # log(1 + e^v) without overflow: max(v, 0) + log1p(e^-|v|)
    return np.maximum(v, 0.0) + np.log1p(np.exp(-np.abs(v)))


def _silu(v: np.ndarray) -> np.ndarray:
    return v / (1.0 + np.exp(-v))


def ssd(x, dt_raw, A_log, B, C, D, dt_bias, z=None, h_in=None, seq_idx=None
        ) -> Tuple[np.ndarray, np.ndarray]:
    """Sequential fp64 Mamba2 scan.

    Shapes: x [Bt, L, H, P]; dt_raw [Bt, L, H]; A_log, D, dt_bias [H]; B, C [Bt, L, G, N]
    with G dividing H; z [Bt, L, H, P] or None; h_in [Bt, H, P, N] or None; seq_idx
    [Bt, L] integers or None.  Activations may be float arrays or bf16 bit patterns
    (uint16), read exactly.  Returns (out [Bt, L, H, P], h_out [Bt, H, P, N]) in fp64.
    """
    x = as_f64(x)
    dtr = as_f64(dt_raw)
    Bm = as_f64(B)
    Cm = as_f64(C)
    Bt, L, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    if H % G:
        raise ValueError("ngroups must divide the number of heads")
    hpg = H // G
    A = -np.exp(np.asarray(A_log, dtype=np.float64))            # [H]
    Dh = np.asarray(D, dtype=np.float64)
    bias = np.asarray(dt_bias, dtype=np.float64)
    zz = None if z is None else as_f64(z)
    h = np.zeros((Bt, H, P, N)) if h_in is None else np.array(h_in, dtype=np.float64)
    out = np.empty((Bt, L, H, P))
    grp = np.arange(H) // hpg                                    # head -> group
    for t in range(L):
        if seq_idx is not None and t > 0:
            reset = np.asarray(seq_idx)[:, t] != np.asarray(seq_idx)[:, t - 1]
            h[reset] = 0.0
        delta = _softplus(dtr[:, t, :] + bias)                   # [Bt, H]
        decay = np.exp(delta * A)                                # [Bt, H]
        Bt_ = Bm[:, t][:, grp, :]                                # [Bt, H, N]
        Ct_ = Cm[:, t][:, grp, :]
        xt = x[:, t]                                             # [Bt, H, P]
        h = decay[:, :, None, None] * h + (delta[:, :, None] * xt)[:, :, :, None] * Bt_[:, :, None, :]
        yt = np.einsum("bhpn,bhn->bhp", h, Ct_) + Dh[None, :, None] * xt
        if zz is not None:
            yt = yt * _silu(zz[:, t])
        out[:, t] = yt
    return out, h


def ssd_channels(x, dt_raw, A_log, B, C, D, dt_bias, sel, z=None, h_in=None, seq_idx=None):
    """The oracle on a subset of (batch row, head) pairs only: ``sel`` is a list of (b, h).

    Each pair is an independent recurrence, so this is the same computation restricted to
    those pairs (used to check large runs on a sample).  Returns lists of out [L, P] and
    h_out [P, N] per pair.
    """
    Bt, L, H, P = x.shape
    G = B.shape[2]
    hpg = H // G
    outs, hs = [], []
    for b, hh in sel:
        g = hh // hpg
        o, hf = ssd(x[b:b + 1, :, hh:hh + 1], dt_raw[b:b + 1, :, hh:hh + 1],
                    np.asarray(A_log)[hh:hh + 1], B[b:b + 1, :, g:g + 1], C[b:b + 1, :, g:g + 1],
                    np.asarray(D)[hh:hh + 1], np.asarray(dt_bias)[hh:hh + 1],
                    None if z is None else z[b:b + 1, :, hh:hh + 1],
                    None if h_in is None else np.asarray(h_in)[b:b + 1, hh:hh + 1],
                    None if seq_idx is None else np.asarray(seq_idx)[b:b + 1])
        outs.append(o[0, :, 0])
        hs.append(hf[0, 0])
    return outs, hs


def conv_silu(xbc, conv_w, conv_b=None, seq_idx=None, conv_state_in=None):
    """The Mamba2 layer's causal depthwise conv + SiLU over the concatenated x, B, C channels
    (niverel-mamba 0.1.0, section "The weight contract": conv1d.weight [channels, 1, 4] and
    conv1d.bias over d_inner + 2 ngroups d_state channels), fp64, one step at a time.

    xbc [Bt, L, Cc] (floats or bf16 bit patterns); conv_w [Cc, K]; conv_b [Cc] or None;
    conv_state_in [Bt, Cc, K - 1] (the K - 1 inputs before step 0, oldest first) or None
    (zeros).  out[b, t, c] = SiLU(conv_b[c] + sum_k conv_w[c, k] * xpad[b, t + k, c]) with
    xpad = [conv state ; xbc] (cross-correlation, left padding; conv_w[c, K - 1] multiplies
    the current input).  With seq_idx, a tap reads zero when an id change lies between its
    input's step and t (the conv state resets where the id changes; the state before step 0
    belongs to the row's first document).  Returns (out [Bt, L,
    Cc], conv_state_out [Bt, Cc, K - 1] = the last K - 1 entries of xpad, zeroed where they
    precede the last document's first step).
    """
    x = as_f64(xbc)
    Bt, L, Cc = x.shape
    w = np.asarray(conv_w, dtype=np.float64)
    K = w.shape[1]
    bias = np.zeros(Cc) if conv_b is None else np.asarray(conv_b, dtype=np.float64)
    st = np.zeros((Bt, Cc, K - 1)) if conv_state_in is None else as_f64(conv_state_in)
    xpad = np.concatenate([np.transpose(st, (0, 2, 1)), x], axis=1)   # [Bt, K-1+L, Cc]
    ids = None if seq_idx is None else np.asarray(seq_idx)
    out = np.empty((Bt, L, Cc))
    for b in range(Bt):
        for t in range(L):
            acc = bias.copy()
            for k in range(K):
                src = t + k - (K - 1)          # time of the tap's input (negative: the state)
                # the tap is dropped when a reset (an id change) lies in (src, t]
                if ids is not None and np.any(ids[b, max(src, 0):t + 1] != ids[b, t]):
                    continue
                acc = acc + w[:, k] * xpad[b, t + k]
            out[b, t] = _silu(acc)
    cs = np.transpose(xpad[:, L:L + K - 1], (0, 2, 1)).copy()         # [Bt, Cc, K-1]
    if ids is not None and L > 0:
        for b in range(Bt):
            for j in range(K - 1):
                src = L - (K - 1) + j          # time of the slot's input (negative: the state)
                if np.any(ids[b, max(src, 0):L] != ids[b, L - 1]):
                    cs[b, :, j] = 0.0
    return out, cs


def gated_rmsnorm(y, z, weight, eps=1e-5, group_size=None):
    """The Mamba2 layer's gated RMSNorm with the gate before the norm (niverel-mamba 0.1.0,
    section "The weight contract": norm.weight over d_inner, eps 1e-5): g = y * SiLU(z);
    out = g / sqrt(mean(g^2) + eps) * weight, the mean over each group of group_size
    consecutive channels (d_inner when None).  y, z [..., d_inner]; fp64."""
    yy = as_f64(y)
    zz = as_f64(z)
    w = np.asarray(weight, dtype=np.float64)
    D = yy.shape[-1]
    gs = D if group_size is None else int(group_size)
    g = yy * _silu(zz)
    gg = g.reshape(g.shape[:-1] + (D // gs, gs))
    r = 1.0 / np.sqrt(np.mean(gg * gg, axis=-1, keepdims=True) + eps)
    return (gg * r).reshape(g.shape) * w
