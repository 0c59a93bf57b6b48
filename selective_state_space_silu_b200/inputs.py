"""Seeded synthetic inputs for the selective-SSM mixer core.

This module draws inputs only.  It holds none of the mixer's arithmetic (no conv,
softplus, scan or gate): the oracle and the CUDA path both take what it returns.

Workloads follow the shapes the pages describe:

* ``tiny``    -- batch 2, L 16, d_inner 128, d_state 16, fp32 I/O.
* ``stress``  -- the openfluke "Apple Mamba stress test" default profile
                 (section "Profiles": d_model 512, expand 2, d_state 8, batch 8,
                 sequence 32), fp32 I/O.
* ``m130``    -- a 130M-class Mamba layer (Octopus Research report, section 1):
                 d_model 768, d_inner 1536, d_state 16, batch 8, L 2048, bf16 I/O.
* ``long``    -- batch 2, L 65536, d_inner 2560, d_state 16, bf16 I/O.
* ``decode``  -- one token for 256 independent sequences, d_inner 5120,
                 d_state 16, bf16 I/O with a cached fp32 state.

Distributions (calm-mamba 0.1.4, section "Mamba operator", names the parameters;
the value recipe is the usual Mamba-1 initialisation):

* x', z, B, C ~ N(0, 1); dt_raw ~ N(0, 0.5) (0.5 is the standard deviation);
* dt_bias = inverse-softplus(dt0) with ln(dt0) ~ U(ln 1e-3, ln 1e-1) per channel;
* A_log[d, n] = ln(n + 1); D = 1; conv_w, conv_b ~ U(-0.5, 0.5);
* decode only: cached h ~ N(0, 1) (fp32), conv state ~ N(0, 1) (I/O dtype).

Draws are made in float32 from ``numpy.random.Generator(PCG64(seed))`` in the order
x', z, dt_raw, B, C, dt_bias, conv_w, conv_b, then h and conv_state, each in C order.
For bf16 workloads every activation is rounded to bf16 (round to nearest even) before
either side sees it, and is kept as its 16-bit pattern (``numpy.uint16``).
"""

from __future__ import annotations

import dataclasses
from typing import Dict, Optional

import numpy as np

F32 = "f32"
BF16 = "bf16"


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    batch: int
    seqlen: int
    d_inner: int
    d_state: int
    d_conv: int
    io_dtype: str          # "f32" or "bf16"
    seed: int
    decode: bool = False   # True: one token on top of a cached state
    packed_mean: int = 0   # > 0: rows pack documents of this mean length (seq_idx)

    @property
    def io_bytes(self) -> int:
        return 4 if self.io_dtype == F32 else 2

    def with_(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


WORKLOADS: Dict[str, Workload] = {
    "tiny": Workload("tiny", 2, 16, 128, 16, 4, F32, 1000),
    "stress": Workload("stress", 8, 32, 1024, 8, 4, F32, 1001),
    "m130": Workload("m130", 8, 2048, 1536, 16, 4, BF16, 1002),
    "long": Workload("long", 2, 65536, 2560, 16, 4, BF16, 1003),
    "decode": Workload("decode", 256, 1, 5120, 16, 4, BF16, 1004, decode=True),
    # the 130M-class layer over rows that pack documents of mean length 256
    "m130_packed": Workload("m130_packed", 8, 2048, 1536, 16, 4, BF16, 1005, packed_mean=256),
}


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (nearest, ties to even); return the 16-bit patterns.

    NaN payloads are kept quiet; infinities stay infinities.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    lsb = (u >> 16) & 1
    r = ((u + 0x7FFF + lsb) >> 16).astype(np.uint16)
    nan = np.isnan(a)
    if nan.any():
        r[nan] = ((u[nan] >> 16) | 0x0040).astype(np.uint16)
    return r


def bf16_bits_to_f32(bits: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns to float32."""
    b = np.ascontiguousarray(bits, dtype=np.uint16)
    return (b.astype(np.uint32) << 16).view(np.float32)


def _normal(rng: np.random.Generator, shape, std: float = 1.0, chunk_rows: int = 1 << 22):
    """N(0, std) float32 draws in C order, in slices of the leading axes (same stream)."""
    out = np.empty(shape, dtype=np.float32)
    flat = out.reshape(-1)
    n = flat.size
    pos = 0
    while pos < n:
        m = min(chunk_rows, n - pos)
        flat[pos:pos + m] = rng.standard_normal(m, dtype=np.float32)
        pos += m
    if std != 1.0:
        flat *= np.float32(std)
    return out


def _act(x: np.ndarray, io_dtype: str) -> np.ndarray:
    return f32_to_bf16_bits(x) if io_dtype == BF16 else x


def make_inputs(w: Workload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw every input of workload ``w``.

    Activations (xp, z, dt_raw, B, C and, for decode, conv_state) come back as float32
    arrays for fp32 workloads and as bf16 bit patterns (uint16) for bf16 workloads.
    Parameters (A_log, D, conv_w, conv_b, dt_bias) and the cached h are float32.
    Layouts: xp, z, dt_raw [batch, L, d_inner]; B, C [batch, L, d_state];
    A_log [d_inner, d_state]; D, conv_b, dt_bias [d_inner]; conv_w [d_inner, d_conv];
    h [batch, d_inner, d_state]; conv_state [batch, d_inner, d_conv - 1] (oldest first).
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    Bt, L, Di, N, K = w.batch, w.seqlen, w.d_inner, w.d_state, w.d_conv
    out: Dict[str, np.ndarray] = {}
    out["xp"] = _act(_normal(rng, (Bt, L, Di)), w.io_dtype)
    out["z"] = _act(_normal(rng, (Bt, L, Di)), w.io_dtype)
    out["dt_raw"] = _act(_normal(rng, (Bt, L, Di), std=0.5), w.io_dtype)
    out["B"] = _act(_normal(rng, (Bt, L, N)), w.io_dtype)
    out["C"] = _act(_normal(rng, (Bt, L, N)), w.io_dtype)
    # dt_bias: dt0 log-uniform on [1e-3, 1e-1]; dt_bias = log(expm1(dt0)) so that the
    # mixer's softplus maps dt_bias back to dt0.
    lo, hi = np.log(1e-3), np.log(1e-1)
    dt0 = np.exp(rng.uniform(lo, hi, size=Di))
    out["dt_bias"] = np.log(np.expm1(dt0)).astype(np.float32)
    out["conv_w"] = rng.uniform(-0.5, 0.5, size=(Di, K)).astype(np.float32)
    out["conv_b"] = rng.uniform(-0.5, 0.5, size=Di).astype(np.float32)
    out["A_log"] = np.tile(np.log(np.arange(1, N + 1, dtype=np.float64)), (Di, 1)).astype(np.float32)
    out["D"] = np.ones(Di, dtype=np.float32)
    if w.decode:
        out["h"] = _normal(rng, (Bt, Di, N))
        out["conv_state"] = _act(_normal(rng, (Bt, Di, K - 1)), w.io_dtype)
    if w.packed_mean > 0:
        out["seq_idx"] = packed_seq_idx(Bt, L, w.packed_mean, (w.seed if seed is None else seed) + 1)
    return out


def make_dtproj_inputs(w: Workload, dt_rank: int, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Inputs of the forward with the dt projection fused: those of ``make_inputs`` (same
    seed, same draws) plus dt_low [batch, L, dt_rank] ~ N(0, 1) and W_dt [d_inner, dt_rank]
    ~ N(0, 0.5^2 / dt_rank), so that dt_low W_dt^T has the N(0, 0.5^2) spread of dt_raw;
    both rounded to bf16 (bit patterns, uint16).  dt_raw is dropped."""
    out = make_inputs(w, seed)
    out.pop("dt_raw")
    rng = np.random.Generator(np.random.PCG64((w.seed if seed is None else seed) + 7777))
    out["dt_low"] = f32_to_bf16_bits(_normal(rng, (w.batch, w.seqlen, dt_rank)))
    out["W_dt"] = f32_to_bf16_bits(_normal(rng, (w.d_inner, dt_rank), std=0.5 / np.sqrt(dt_rank)))
    return out


def random_params(w: Workload, seed: int) -> Dict[str, np.ndarray]:
    """Random A_log and D (instead of the structured ln(1..N) and 1) for extra cases."""
    rng = np.random.Generator(np.random.PCG64(seed))
    Di, N = w.d_inner, w.d_state
    return {
        "A_log": rng.uniform(-1.0, 3.0, size=(Di, N)).astype(np.float32),
        "D": rng.standard_normal(Di, dtype=np.float32),
    }


def as_f64(a: np.ndarray) -> np.ndarray:
    """Exact float64 view of an activation as either side reads it."""
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a).astype(np.float64)
    return np.asarray(a, dtype=np.float64)


def as_f32(a: np.ndarray) -> np.ndarray:
    if a.dtype == np.uint16:
        return bf16_bits_to_f32(a)
    return np.asarray(a, dtype=np.float32)


# ---------------------------------------------------------------- packed documents
# seq_idx patterns for rows that pack several documents (niverel-mamba 0.1.0, section
# "seq_idx strict reset": the states reset wherever seq_idx changes).  The nine shapes
# follow the structural cases that section lists; they are index patterns only.
SEQ_IDX_CASES = ("start_of_row", "length_one_docs", "consecutive_boundaries", "boundary_on_edge",
                 "doc_inside_chunk", "misaligned_rows", "terminal_padding", "nonzero_first_id",
                 "many_short_docs")


def _runs_to_ids(lengths, first_id: int = 0) -> np.ndarray:
    return np.repeat(np.arange(first_id, first_id + len(lengths)), lengths).astype(np.int32)


def _row(L: int, cuts, first_id: int = 0) -> np.ndarray:
    """Ids for one row with documents starting at the given positions (besides 0)."""
    cuts = sorted(c for c in set(cuts) if 0 < c < L)
    bounds = [0] + cuts + [L]
    return _runs_to_ids(np.diff(bounds), first_id)


def seq_idx_case(name: str, batch: int, L: int, edge: int = 8, seed: int = 0) -> np.ndarray:
    """One of SEQ_IDX_CASES as an int32 [batch, L] array.  ``edge`` is a block length of
    the implementation (a tile or chunk length) for the boundary-on-edge case."""
    r = np.random.default_rng(seed)
    rows = []
    for b in range(batch):
        if name == "start_of_row":            # every row opens a new id; no other boundary
            row = np.full(L, 100 + 7 * b, dtype=np.int32)
        elif name == "length_one_docs":
            row = _row(L, [1, 2, 3, L // 2, L // 2 + 1, L - 1], first_id=b)
        elif name == "consecutive_boundaries":
            m = L // 3 + b
            row = _row(L, [m, m + 1, m + 2, m + 3])
        elif name == "boundary_on_edge":
            row = _row(L, [k * edge for k in range(1, L // edge + 1)][: 4 + b])
        elif name == "doc_inside_chunk":
            a = max(1, L // 2 - 3 + b)
            row = _row(L, [a, a + 5])
        elif name == "misaligned_rows":
            row = _row(L, sorted(r.choice(np.arange(1, L), size=min(L - 1, 3 + b), replace=False)))
        elif name == "terminal_padding":
            pad = max(1, L // 5)
            row = _row(L, [L // 3 + b, L - pad])
            row[L - pad:] = -1
        elif name == "nonzero_first_id":
            row = _row(L, [L // 4 + b], first_id=42)
        elif name == "many_short_docs":
            lens = []
            while sum(lens) < L:
                lens.append(int(r.integers(1, 6)))
            row = _runs_to_ids(lens)[:L]
        else:
            raise ValueError(name)
        rows.append(row.astype(np.int32))
    return np.stack(rows)


def packed_seq_idx(batch: int, L: int, mean_len: int, seed: int) -> np.ndarray:
    """Rows packing documents of geometric length (mean ``mean_len``), for timing."""
    r = np.random.default_rng(seed)
    out = np.empty((batch, L), dtype=np.int32)
    for b in range(batch):
        lens = []
        while sum(lens) < L:
            lens.append(int(r.geometric(1.0 / mean_len)))
        out[b] = _runs_to_ids(lens)[:L]
    return out


# ---------------------------------------------------------------- Mamba2 (SSD) scan
# niverel-mamba 0.1.0, section "The weight contract": the reference layer has d_model 768,
# expand 2 (1536 inner channels = 24 heads of headdim 64), d_state 128, ngroups 1, and
# dt_bias, A_log and D of one value per head.
@dataclasses.dataclass(frozen=True)
class SsdWorkload:
    name: str
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    d_state: int
    ngroups: int
    seed: int
    gate: bool = False      # draw z (the y * SiLU(z) gate of the rmsnorm=False layer)
    state: bool = False     # draw an initial state h_in


SSD_WORKLOADS: Dict[str, SsdWorkload] = {
    "ssd_tiny": SsdWorkload("ssd_tiny", 2, 100, 4, 64, 64, 1, 2000, gate=True),
    # the reference layer (24 heads x 64, d_state 128) over 8 rows of 2048 tokens
    "ssd_v3": SsdWorkload("ssd_v3", 8, 2048, 24, 64, 128, 1, 2001),
    # the same layer over 2 rows of 8192 tokens (the length the pages certify resets at)
    "ssd_v3_long": SsdWorkload("ssd_v3_long", 2, 8192, 24, 64, 128, 1, 2002),
    # one decode step of the same layer for 256 sequences on cached states (gated)
    "ssd_v3_decode": SsdWorkload("ssd_v3_decode", 256, 1, 24, 64, 128, 1, 2003, gate=True, state=True),
}


def make_ssd_inputs(w: SsdWorkload, seed: Optional[int] = None) -> Dict[str, np.ndarray]:
    """Draw every input of Mamba2 scan workload ``w`` (activations as bf16 bit patterns).

    Layouts: x, z [batch, L, nheads, headdim]; dt_raw [batch, L, nheads]; B, C [batch, L,
    ngroups, d_state]; A_log, D, dt_bias [nheads]; h_in [batch, nheads, headdim, d_state].
    Draw order x, dt_raw, B, C, then z, dt_bias, A, h_in (PCG64(seed), float32):
    x, B, C, z ~ N(0, 1) (x stands in for the post-conv activation); dt_raw ~ N(0, 0.5);
    dt0 log-uniform on [1e-3, 1e-1] per head and dt_bias = log(expm1(dt0)); A ~ U(1, 16)
    per head and A_log = ln(A); D = 1; h_in ~ N(0, 1) fp32.
    """
    rng = np.random.Generator(np.random.PCG64(w.seed if seed is None else seed))
    Bt, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.d_state, w.ngroups
    out: Dict[str, np.ndarray] = {}
    out["x"] = f32_to_bf16_bits(_normal(rng, (Bt, L, H, P)))
    out["dt_raw"] = f32_to_bf16_bits(_normal(rng, (Bt, L, H), std=0.5))
    out["B"] = f32_to_bf16_bits(_normal(rng, (Bt, L, G, N)))
    out["C"] = f32_to_bf16_bits(_normal(rng, (Bt, L, G, N)))
    out["z"] = f32_to_bf16_bits(_normal(rng, (Bt, L, H, P))) if w.gate else None
    lo, hi = np.log(1e-3), np.log(1e-1)
    dt0 = np.exp(rng.uniform(lo, hi, size=H))
    out["dt_bias"] = np.log(np.expm1(dt0)).astype(np.float32)
    out["A_log"] = np.log(rng.uniform(1.0, 16.0, size=H)).astype(np.float32)
    out["D"] = np.ones(H, dtype=np.float32)
    out["h_in"] = _normal(rng, (Bt, H, P, N)) if w.state else None
    return out
