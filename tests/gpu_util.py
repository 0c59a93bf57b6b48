"""Helpers shared by the GPU parity tests: move seeded inputs to the device, run the
C-ABI entry points through the binding, and run the oracle on the same inputs."""

from __future__ import annotations

import numpy as np
import torch

from selective_state_space_silu_b200 import inputs as I

ACT = ("xp", "z", "dt_raw", "B", "C")
PARAMS = ("A_log", "D", "conv_w", "conv_b", "dt_bias")


def dev_tensor(a: np.ndarray, device="cuda") -> torch.Tensor:
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host(t: torch.Tensor) -> np.ndarray:
    if t.dtype == torch.bfloat16:
        return t.float().cpu().numpy().astype(np.float64)
    return t.cpu().numpy().astype(np.float64)


def host_bits(t: torch.Tensor) -> np.ndarray:
    """Raw storage of a device tensor (bf16 as uint16 patterns, fp32 as float32)."""
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).cpu().numpy().view(np.uint16)
    return t.cpu().numpy()


def to_device(inp: dict, device="cuda") -> dict:
    out = {}
    for k, v in inp.items():
        out[k] = None if v is None else dev_tensor(v, device)
    return out


def gpu_fwd(d: dict, **kw):
    from selective_state_space_silu_b200.mixer import mamba_mixer_fwd
    return mamba_mixer_fwd(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                           d["conv_w"], d.get("conv_b"), d["dt_bias"], **kw)


def gpu_step(d: dict, h_in, cs_in, **kw):
    from selective_state_space_silu_b200.mixer import mamba_mixer_step
    return mamba_mixer_step(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                            d["conv_w"], d.get("conv_b"), d["dt_bias"], h_in, cs_in, **kw)


def oracle_full(oracle, inp: dict, with_state=False, nthreads=0):
    w = I.as_f64
    return oracle.mixer(w(inp["xp"]), w(inp["z"]), w(inp["dt_raw"]), w(inp["B"]), w(inp["C"]),
                        inp["A_log"], inp["D"], inp["conv_w"], inp.get("conv_b"), inp["dt_bias"],
                        inp.get("h") if with_state else None,
                        w(inp["conv_state"]) if with_state else None, nthreads=nthreads)


def pick_channels(Di: int, n: int, seed: int) -> np.ndarray:
    """Sampled channels: both ends, tile edges, and random ones."""
    r = np.random.default_rng(seed)
    edges = [0, 1, 7, 8, 31, 32, 127, 128, Di // 2, Di - 129, Di - 128, Di - 1]
    pick = set(e for e in edges if 0 <= e < Di)
    while len(pick) < min(n, Di):
        pick.add(int(r.integers(0, Di)))
    return np.array(sorted(pick))
