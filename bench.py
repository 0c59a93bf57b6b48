#!/usr/bin/env python
"""Benchmark of the fused selective-SSM mixer core on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload m130|long|decode|stress|tiny]

One step = one pass of the whole hot path over one batch: the fused forward
(conv+SiLU, softplus, selective scan with the chunk carry, gate, state out) over the
workload's prompt, then one decode step per sequence on the state the forward left
(in place).  The default workload is the long-sequence one (batch 2, L 65536, d_inner
2560): the only one whose forward also runs the carry between time chunks, so its step
covers every stage of the path.  ``--workload decode`` times the decode step alone.

Prints ONE JSON line (rank 0).  ``value`` is achieved algorithmic HBM GB/s over all
ranks: algorithmic bytes (each input read once, each output written once) divided by
the device time of the K timed steps (CUDA events on the launching stream, L2 flushed
between steps, max over ranks).  ``--impl reference`` times the CPU oracle instead.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from selective_state_space_silu_b200 import inputs as I  # noqa: E402

METRIC = "fused conv+selective-scan+gate: achieved HBM GB/s and % of B200 peak"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- bytes
def fwd_bytes(w: I.Workload) -> int:
    s = w.io_bytes
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    return (4 * Bt * L * Di * s            # x', z, dt_raw in; y out
            + 2 * Bt * L * N * s           # B, C
            + Di * (4 * N + 28)            # A_log, D, conv_w, conv_b, dt_bias
            + Bt * Di * N * 4              # h out
            + Bt * Di * 3 * s              # conv state out
            + (4 * Bt * L if w.packed_mean else 0))   # seq_idx


def step_bytes(w: I.Workload) -> int:
    s = w.io_bytes
    Bt, Di, N = w.batch, w.d_inner, w.d_state
    return (Bt * Di * (2 * N * 4 + 2 * 3 * s + 4 * s)   # h in/out, conv state in/out, x' z dt y
            + 2 * Bt * N * s                          # B, C of the token
            + Di * (4 * N + 28))


def workload_bytes(w: I.Workload) -> dict:
    if w.decode:
        return {"fwd": 0, "step": step_bytes(w)}
    return {"fwd": fwd_bytes(w), "step": step_bytes(w.with_(seqlen=1))}


# ----------------------------------------------------------------------------- rooflines
SMS = 148
MUFU_PER_CLK_SM = 16      # special-function (ex2/lg2/rcp) lane-ops per clock per SM
FMA_PER_CLK_SM = 128      # fp32 FMA-pipe lane-ops per clock per SM
POLY_EXP_FMA_OPS = 9      # FMA-pipe ops for one exp done by polynomial instead of MUFU


def alu_elements_per_clk_sm(N: int) -> float:
    """Upper bound on scan elements (t, d, n) per clock per SM from the arithmetic alone.

    Per element the method needs T = 1 + 4/N transcendentals (exp(Delta*A) per state, and
    per (t, d) the exps of the two SiLUs and the exp + log of softplus) and F = 4 + 20/N
    fp32 ops (Delta*A, Delta*u*B, the h FMA, the C.h FMA; per (t, d) about 20 for the conv,
    gate and the arithmetic around the transcendentals).  Transcendentals go to MUFU (16 per
    clock per SM) or, as a degree-5 polynomial, to the FMA pipe (9 ops each).  With MUFU
    saturated and the rest of the transcendentals on the FMA pipe:
        F*x + 9*(T*x - 16) = 128   ->   x = (128 + 9*16) / (F + 9*T).
    """
    T = 1.0 + 4.0 / N
    F = 4.0 + 20.0 / N
    x = (FMA_PER_CLK_SM + POLY_EXP_FMA_OPS * MUFU_PER_CLK_SM) / (F + POLY_EXP_FMA_OPS * T)
    if T * x < MUFU_PER_CLK_SM:          # MUFU alone suffices; the FMA pipe binds
        x = FMA_PER_CLK_SM / F
    return x


def alu_floor_s(elements: int, N: int, sm_hz: float) -> float:
    return elements / (alu_elements_per_clk_sm(N) * SMS * sm_hz)


# ----------------------------------------------------------------------------- ranks
def max_over_ranks(x: float, dist=None, device=None) -> float:
    """The largest x over all ranks (the job's time is its slowest rank's time)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_gbs(bytes_per_rank_step: int, steps: int, world: int, max_ms: float) -> float:
    """Whole-job throughput: every rank moves bytes_per_rank_step per step (weak scaling);
    the job takes as long as its slowest rank."""
    return world * bytes_per_rank_step * steps / (max_ms * 1e-3) / 1e9


# ----------------------------------------------------------------------------- misc
FALLBACK_BF16_TFLOPS = 1590.0   # an earlier cuBLAS bf16 burst on this pool


def peak_labels(peaks: dict):
    """(HBM, bf16) peak sources as the JSON line states them: measured, or the fallback."""
    hbm = ("measured (MEASURED_PEAKS.json hbm_gbs)" if peaks.get("source") == "measured"
           else f"fallback {FALLBACK_HBM_GBS:.0f} GB/s")
    bf16 = ("measured cuBLAS bf16 burst (MEASURED_PEAKS.json bf16_tflops)"
            if peaks.get("bf16_source") == "measured"
            else f"fallback {FALLBACK_BF16_TFLOPS:.0f} TFLOP/s (earlier cuBLAS bf16 burst)")
    return hbm, bf16


def measured_peaks() -> dict:
    """The measured peaks (HBM copy GB/s; cuBLAS bf16 burst TFLOP/s, for kernels timed
    alone) when MEASURED_PEAKS.json is present, else the fallback figures."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    out = {"hbm_gbs": FALLBACK_HBM_GBS, "source": "fallback",
           "bf16_tflops": FALLBACK_BF16_TFLOPS, "bf16_source": "fallback"}
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        if d.get("hbm_gbs"):
            out["hbm_gbs"], out["source"] = float(d["hbm_gbs"]), "measured"
        if d.get("bf16_tflops"):
            out["bf16_tflops"], out["bf16_source"] = float(d["bf16_tflops"]), "measured"
    return out


# The files that define each entry point's kernels; a recorded traffic figure is used only
# while they are unchanged.  (Host code and the time-chunk plan live in mamba_mixer.cu; each
# record names the plan it was taken with.)
KERNEL_SOURCES = {
    "fwd": ("fwd_kernel.cuh", "fwd2_kernel.cuh", "device_math.cuh", "sm100_primitives.cuh"),
    "step": ("step.cuh", "device_math.cuh", "sm100_primitives.cuh"),
    "ssd": ("ssd_kernel.cuh", "ssd_tc_kernel.cuh", "device_math.cuh", "sm100_primitives.cuh"),
    "ssd_step": ("ssd_step.cuh", "device_math.cuh"),
}


def kernel_source_hash(kind: str) -> str:
    """Hash of the code (comments and blank lines dropped) of the sources that define one
    entry point's kernels, so that a recorded traffic figure survives comment edits only."""
    import re
    h = hashlib.sha256()
    for name in KERNEL_SOURCES[kind]:
        with open(os.path.join(ROOT, "selective_state_space_silu_b200", "csrc", name)) as fh:
            text = fh.read()
        code = [re.sub(r"//.*$", "", line).rstrip() for line in text.splitlines()]
        h.update(name.encode() + b"\0" + "\n".join(l for l in code if l).encode())
    return h.hexdigest()[:16]


def recorded_traffic(kind: str, workload: str):
    """DRAM bytes (read + write) per call of the dominant entry point, from the committed
    ncu summary profiles/<kind>_<workload>_traffic.txt, if those counters were taken on the
    current kernel sources; else None."""
    p = os.path.join(ROOT, "profiles", f"{kind}_{workload}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    for line in open(p):
        if ":" in line:
            k, v = line.split(":", 1)
            kv[k.strip()] = v.strip()
    if kv.get("kernel_source_sha") != kernel_source_hash(kind):
        return None
    try:
        return int(float(kv["dram_bytes_per_call"]))
    except (KeyError, ValueError):
        return None


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed region runs."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.index}", f"--query-gpu={self.Q}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        return self

    def __exit__(self, *a):
        self.out = ""
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.out, _ = self.proc.communicate(timeout=10)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.out, _ = self.proc.communicate()

    def summary(self) -> dict:
        rows = []
        for line in (self.out or "").strip().splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append({"sm": float(parts[1]), "max": float(parts[2]),
                             "hw": parts[5], "hwt": parts[6], "swt": parts[7], "pc": parts[8]})
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        load = [r for r in rows if r["sm"] > 0.5 * r["max"]] or rows
        reasons = set()
        for r in rows:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pc", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load),
                "sm_max_mhz": max(r["max"] for r in rows), "reasons": sorted(reasons),
                "samples": len(rows)}


# ----------------------------------------------------------------------------- ours
def run_ours(args, w: I.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    from selective_state_space_silu_b200 import mixer as M

    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M.load_library()
    inp = I.make_inputs(w)
    tok_w = w.with_(seqlen=1, decode=True, seed=w.seed + 7919)
    tok = I.make_inputs(tok_w)     # the decode token (its h / conv_state are unused)

    def td(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    P = {k: td(inp[k]) for k in ("A_log", "D", "conv_w", "conv_b", "dt_bias")}
    X = {k: td(inp[k]) for k in ("xp", "z", "dt_raw", "B", "C")}
    if w.packed_mean:
        X["seq_idx"] = td(inp["seq_idx"])
    T = {k: td(tok[k]) for k in ("xp", "z", "dt_raw", "B", "C")}
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    iot = X["xp"].dtype
    stream = torch.cuda.current_stream(dev)
    if w.decode:
        h = td(inp["h"])
        cs = td(inp["conv_state"])
        y = torch.empty((Bt, 1, Di), dtype=iot, device=dev)
        ws = None
        X = T = {k: td(inp[k]) for k in ("xp", "z", "dt_raw", "B", "C")}
    else:
        y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
        h = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
        cs = torch.empty((Bt, Di, 3), dtype=iot, device=dev)
        ws = M.new_workspace(M.make_dims(Bt, L, Di, N, 4, M._io_code(X["xp"])), dev)
    yt = torch.empty((Bt, 1, Di), dtype=iot, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():
        # write a buffer larger than L2, then read another one: the timed kernels start
        # with a cold L2 holding clean lines (no write-back of the flush inside the timing)
        flush.fill_(1.0)
        torch.sum(flush_rd, dim=0, out=flush_sink)

    def fwd():
        if w.packed_mean:
            M.mamba_mixer_fwd_packed(X["xp"], X["z"], X["dt_raw"], X["B"], X["C"], P["A_log"],
                                     P["D"], P["conv_w"], P["conv_b"], P["dt_bias"],
                                     seq_idx=X["seq_idx"], y=y, h_out=h, conv_state_out=cs,
                                     workspace=ws, stream=stream)
            return
        M.mamba_mixer_fwd(X["xp"], X["z"], X["dt_raw"], X["B"], X["C"], P["A_log"], P["D"],
                          P["conv_w"], P["conv_b"], P["dt_bias"], y=y, h_out=h,
                          conv_state_out=cs, workspace=ws, stream=stream)

    def step():
        M.mamba_mixer_step(T["xp"], T["z"], T["dt_raw"], T["B"], T["C"], P["A_log"], P["D"],
                           P["conv_w"], P["conv_b"], P["dt_bias"], h, cs, y=yt, h_out=h,
                           conv_state_out=cs, stream=stream)

    launches_fwd = 0 if w.decode else M.mamba_mixer_fwd_launches(M.make_dims(Bt, L, Di, N, 4, M._io_code(X["xp"])))
    launches_per_step = launches_fwd + 1

    def one_step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        if not w.decode:
            fwd()
        if ev is not None:
            ev[1].record(stream)
        step()
        if ev is not None:
            ev[2].record(stream)

    for _ in range(args.warmup):
        flush_l2()
        one_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for i in range(args.steps):
            flush_l2()              # not timed
            one_step(evs[i])
        torch.cuda.synchronize()
    step_ms = [e[0].elapsed_time(e[2]) for e in evs]
    fwd_ms = [e[0].elapsed_time(e[1]) for e in evs]
    dec_ms = [e[1].elapsed_time(e[2]) for e in evs]
    total_ms = max_over_ranks(sum(step_ms), dist if world > 1 else None, dev)
    if world > 1:
        dist.barrier()

    # end to end through the public API: pinned host inputs -> device -> mixer -> host
    e2e = None
    if rank == 0 or world > 1:
        hx = {k: v.cpu().pin_memory() for k, v in X.items()}
        ht = {k: v.cpu().pin_memory() for k, v in T.items()}
        hy = torch.empty(y.shape, dtype=iot).pin_memory()
        hyt = torch.empty(yt.shape, dtype=iot).pin_memory()
        hh = torch.empty(h.shape, dtype=torch.float32).pin_memory()
        hcs = torch.empty(cs.shape, dtype=iot).pin_memory()
        h2d = sum(v.numel() * v.element_size() for v in hx.values())
        if not w.decode:
            h2d += sum(v.numel() * v.element_size() for v in ht.values())
        d2h = (0 if w.decode else hy.numel() * hy.element_size()) + hyt.numel() * hyt.element_size() \
            + hh.numel() * 4 + hcs.numel() * hcs.element_size()
        if w.decode:
            h2d += hh.numel() * 4 + hcs.numel() * hcs.element_size()
            hh0, hcs0 = h.cpu().pin_memory(), cs.cpu().pin_memory()
        e2e_steps = max(3, min(args.steps, 50))
        ev0 = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
        ev1 = [torch.cuda.Event(enable_timing=True) for _ in range(e2e_steps)]
        for i in range(e2e_steps + 2):
            flush_l2()
            if i >= 2:
                ev0[i - 2].record(stream)
            for k in X:
                X[k].copy_(hx[k], non_blocking=True)
            if not w.decode:
                for k in T:
                    T[k].copy_(ht[k], non_blocking=True)
            else:
                h.copy_(hh0, non_blocking=True)
                cs.copy_(hcs0, non_blocking=True)
            one_step()
            if not w.decode:
                hy.copy_(y, non_blocking=True)
            hyt.copy_(yt, non_blocking=True)
            hh.copy_(h, non_blocking=True)
            hcs.copy_(cs, non_blocking=True)
            if i >= 2:
                ev1[i - 2].record(stream)
        torch.cuda.synchronize()
        e2e_ms = max_over_ranks(sum(a.elapsed_time(b) for a, b in zip(ev0, ev1)),
                                dist if world > 1 else None, dev)
        e2e = {"ms_per_step": e2e_ms / e2e_steps, "h2d": h2d, "d2h": d2h}

    bytes_ = workload_bytes(w)
    step_total = bytes_["fwd"] + bytes_["step"]
    if rank != 0:
        return None
    # outputs of one clean call (outside the timing) for the parity sample
    if w.decode:
        h.copy_(td(inp["h"]))
        cs.copy_(td(inp["conv_state"]))
        hs = torch.empty_like(h)
        css = torch.empty_like(cs)
        M.mamba_mixer_step(T["xp"], T["z"], T["dt_raw"], T["B"], T["C"], P["A_log"], P["D"],
                           P["conv_w"], P["conv_b"], P["dt_bias"], h, cs, y=yt, h_out=hs,
                           conv_state_out=css, stream=stream)
        outs = (yt, hs, css)
    else:
        fwd()
        outs = (y, h, cs)
    torch.cuda.synchronize()
    peaks = measured_peaks()
    value = job_gbs(step_total, args.steps, world, total_ms)
    # dominant kernel: the forward call (the decode step when timing decode alone)
    if w.decode:
        dom_ms = statistics.mean(dec_ms)
        dom_bytes = bytes_["step"]
        dom = "mamba_mixer_step"
    else:
        dom_ms = statistics.mean(fwd_ms)
        dom_bytes = bytes_["fwd"]
        dom = "mamba_mixer_fwd_packed" if w.packed_mean else "mamba_mixer_fwd"
    clocks = clk.summary()
    sm_hz = (clocks.get("sm_max_mhz") or 1965.0) * 1e6
    roof = roofline_of("step" if w.decode else "fwd", w, dom_bytes, dom_ms, peaks, sm_hz, dom)
    e2e_val = job_gbs(step_total, 1, world, e2e["ms_per_step"])
    return {
        "metric": METRIC,
        "value": round(value, 2),
        "unit": "GB/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(total_ms / args.steps, 5),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16" if w.io_dtype == I.BF16 else "f32",
        "data": "synthetic (seeded; shapes and distributions of the pages' workloads)",
        "config": {
            "workload": w.name,
            "batch": w.batch, "seqlen": w.seqlen, "d_inner": w.d_inner, "d_state": w.d_state,
            "d_conv": w.d_conv, "io": w.io_dtype, "state": "f32",
            "step": ("decode step only" if w.decode else
                     "fused forward over the prompt + one decode step (state in place)"),
            "documents": (f"packed, mean length {w.packed_mean} (seq_idx resets)"
                          if w.packed_mean else None),
            "global_batch": w.batch * world,
            "parallelism": f"replicas x{world} (independent sequences per GPU, no collective)",
            "l2": "flushed between timed steps (256 MiB write + 256 MiB read, outside the timed events)",
            "algorithmic_bytes_per_step": step_total,
        },
        "tokens_channels_per_s": round(world * w.batch * w.seqlen * w.d_inner * args.steps
                                        / (total_ms * 1e-3), 1),
        "fwd_ms_mean": round(statistics.mean(fwd_ms), 5) if not w.decode else None,
        "decode_ms_mean": round(statistics.mean(dec_ms), 5),
        "roofline": roof,
        "e2e": {"value": round(e2e_val, 2), "unit": "GB/s",
                "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                "ms_per_step": round(e2e["ms_per_step"], 4)},
        "gpu_launches": launches_per_step * args.steps if not w.decode else args.steps,
        "clocks": clocks,
        "_outs": (inp, outs),
    }


# ----------------------------------------------------------------------------- parity
def parity_report(got: np.ndarray, ref: np.ndarray, io: str, rounded_io: bool) -> dict:
    """Agreement of device results with the fp64 oracle, in the openfluke stress test's
    terms (section "What the results mean"): the share within the sealed tolerance class,
    the share of exact bits, max abs / rel error; non-finite values count as errors.
    ``rounded_io``: the device result is stored in the I/O type, so "exact" compares it with
    the oracle value rounded to that type (round to nearest even, via fp32)."""
    from tests.tolerances import report
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    r = report(got, ref, io)
    if rounded_io and io == I.BF16:
        rb = I.bf16_bits_to_f32(I.f32_to_bf16_bits(ref.astype(np.float32))).astype(np.float64)
    else:
        rb = ref.astype(np.float32).astype(np.float64)
    exact = float((got == rb).mean()) * 100.0 if got.size else 100.0
    return {"n": r["n"], "within_pct": round(r["within_pct"], 4), "exact_pct": round(exact, 3),
            "max_abs": float(f"{r['max_abs']:.3e}"), "max_rel": float(f"{r['max_rel']:.3e}"),
            "nonfinite": int((~np.isfinite(got)).sum())}


def parity_of(w: I.Workload, inp: dict, y, h, cs, chans, oracle_out=None) -> dict:
    """Compares the device outputs (torch tensors of the whole workload) on the sampled
    channels (all batch rows) with the oracle run on those channels."""
    from oracle import mixer_oracle as O
    if oracle_out is None:
        oracle_out = O.mixer_channels(inp, np.arange(w.batch), chans, widen=I.as_f64, nthreads=0)
    yo, ho, cso = oracle_out
    yg = y.float().cpu().numpy()[:, :, chans]
    hg = h.cpu().numpy()[:, chans]
    cg = cs.float().cpu().numpy()[:, chans]
    return {"sample": f"all {w.batch} batch rows x {len(chans)} of {w.d_inner} channels x L={w.seqlen}",
            "tolerance": w.io_dtype,
            "y": parity_report(yg, yo, w.io_dtype, True),
            "h": parity_report(hg, ho, w.io_dtype, False),
            "conv_state_bitwise": bool(np.array_equal(cg, cso.astype(np.float32)))}


def roofline_of(kind: str, w: I.Workload, dom_bytes: int, dom_ms: float, peaks: dict,
                sm_hz: float, kernel: str) -> dict:
    """The binding roofline of one entry point's call: HBM bytes or the ALU floor."""
    achieved = dom_bytes / (dom_ms * 1e-3) / 1e9
    t_hbm = dom_bytes / (peaks["hbm_gbs"] * 1e9)
    elems = w.batch * (1 if w.decode else w.seqlen) * w.d_inner * w.d_state
    t_alu = alu_floor_s(elems, w.d_state, sm_hz)
    src = peak_labels(peaks)[0]
    if t_alu > t_hbm:
        roof = {"kernel": kernel, "bound": "alu", "achieved": round(achieved, 2),
                "peak": round(dom_bytes / t_alu / 1e9, 2), "unit": "GB/s",
                "frac": round(t_alu / (dom_ms * 1e-3), 4),
                "peak_source": (f"arithmetic floor: {alu_elements_per_clk_sm(w.d_state):.2f} scan "
                                f"elements/clk/SM (MUFU 16 + FMA 128 per clk per SM) x {SMS} SMs x "
                                f"{sm_hz/1e6:.0f} MHz, as GB/s of the kernel's algorithmic bytes"),
                "hbm_frac": round(achieved / peaks["hbm_gbs"], 4),
                "hbm_peak": peaks["hbm_gbs"], "hbm_peak_source": src}
    else:
        roof = {"kernel": kernel, "bound": "hbm", "achieved": round(achieved, 2),
                "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(achieved / peaks["hbm_gbs"], 4), "peak_source": src}
    roof["traffic"] = recorded_traffic(kind, w.name)
    roof["algorithmic_bytes_per_launch"] = dom_bytes
    roof["avg_launch_ms"] = round(dom_ms, 5)
    return roof


def measure_extra(w: I.Workload, dev, calls: int, peaks: dict, n_chans: int) -> dict:
    """One more configuration on this GPU, outside the headline step: ``calls`` forward
    calls (or decode steps) timed one by one with CUDA events on the launching stream, L2
    flushed before each; then one call's outputs against the oracle on sampled channels."""
    import torch
    from selective_state_space_silu_b200 import mixer as M

    inp = I.make_inputs(w)

    def td(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    d = {k: td(v) for k, v in inp.items()}
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    stream = torch.cuda.current_stream(dev)
    iot = d["xp"].dtype
    y = torch.empty((Bt, L, Di), dtype=iot, device=dev)
    h = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    cs = torch.empty((Bt, Di, 3), dtype=iot, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush_l2():   # as in the headline loop: a write, then a read, so L2 holds clean lines
        flush.fill_(1.0)
        torch.sum(flush_rd, dim=0, out=sink)

    if w.decode:
        kernel = "mamba_mixer_step"
        nbytes = step_bytes(w)

        def call():
            M.mamba_mixer_step(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                               d["conv_w"], d["conv_b"], d["dt_bias"], d["h"], d["conv_state"],
                               y=y, h_out=h, conv_state_out=cs, stream=stream)
    else:
        kernel = "mamba_mixer_fwd"
        nbytes = fwd_bytes(w)
        ws = M.new_workspace(M.make_dims(Bt, L, Di, N, 4, M._io_code(d["xp"])), dev)

        def call():
            M.mamba_mixer_fwd(d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"],
                              d["conv_w"], d["conv_b"], d["dt_bias"], y=y, h_out=h,
                              conv_state_out=cs, workspace=ws, stream=stream)
    for _ in range(5):
        flush_l2()
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(calls)]
    with ClockSampler(dev.index or 0) as clk:
        for a, b in evs:
            flush_l2()
            a.record(stream)
            call()
            b.record(stream)
        torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    clocks = clk.summary()
    sm_hz = (clocks.get("sm_max_mhz") or 1965.0) * 1e6
    call()
    torch.cuda.synchronize()
    from tests.gpu_util import pick_channels
    chans = pick_channels(Di, n_chans, w.seed)
    return {"config": {"batch": Bt, "seqlen": L, "d_inner": Di, "d_state": N, "io": w.io_dtype,
                       "entry_point": kernel},
            "calls": calls, "ms": round(ms, 5), "gbs": round(nbytes / (ms * 1e-3) / 1e9, 2),
            "hbm_frac": round(nbytes / (ms * 1e-3) / 1e9 / peaks["hbm_gbs"], 4),
            "roofline": roofline_of("step" if w.decode else "fwd", w, nbytes, ms, peaks, sm_hz,
                                    kernel),
            "parity": parity_of(w, inp, y, h, cs, chans),
            "clocks": clocks}


# ----------------------------------------------------------------------------- dt proj
def dtproj_rank(w: I.Workload) -> int:
    """dt_rank of the workload's model: ceil(d_model / 16) with d_model = d_inner / 2 (the
    calm-mamba layer: expand 2, dt_rank 'auto'), rounded up to a multiple of 8."""
    r = -(-(w.d_inner // 2) // 16)
    return -(-r // 8) * 8


def run_dtproj(args, w: I.Workload, local_rank: int):
    """--pass dtproj: the forward with the dt projection fused (mamba_mixer_fwd_dtproj)
    against the unfused pair (dt_proj as a cuBLAS bf16 GEMM through torch, then
    mamba_mixer_fwd), both timed with CUDA events, L2 flushed before each call."""
    import torch
    from selective_state_space_silu_b200 import mixer as M
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M.load_library()
    R = dtproj_rank(w)
    inp = I.make_dtproj_inputs(w, R)

    def td(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    d = {k: td(v) for k, v in inp.items()}
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    stream = torch.cuda.current_stream(dev)
    y = torch.empty((Bt, L, Di), dtype=torch.bfloat16, device=dev)
    h = torch.empty((Bt, Di, N), dtype=torch.float32, device=dev)
    cs = torch.empty((Bt, Di, 3), dtype=torch.bfloat16, device=dev)
    dt_raw = torch.empty((Bt, L, Di), dtype=torch.bfloat16, device=dev)
    ws = M.new_workspace(M.make_dims(Bt, L, Di, N, 4, M.MAMBA_BF16), dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    def fused():
        M.mamba_mixer_fwd_dtproj(d["xp"], d["z"], d["dt_low"], d["W_dt"], d["B"], d["C"],
                                 d["A_log"], d["D"], d["conv_w"], d["conv_b"], d["dt_bias"],
                                 y=y, h_out=h, conv_state_out=cs, workspace=ws, stream=stream)

    def unfused():
        torch.matmul(d["dt_low"], d["W_dt"].t(), out=dt_raw)
        M.mamba_mixer_fwd(d["xp"], d["z"], dt_raw, d["B"], d["C"], d["A_log"], d["D"],
                          d["conv_w"], d["conv_b"], d["dt_bias"], y=y, h_out=h,
                          conv_state_out=cs, workspace=ws, stream=stream)

    def timed(fn, n):
        for _ in range(args.warmup):
            flush.fill_(1.0)
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for a, b in evs:
            flush.fill_(1.0)
            a.record(stream)
            fn()
            b.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    n = min(args.steps, 50 if w.seqlen > 8192 else 200)
    with ClockSampler(local_rank) as clk:
        ms_f = timed(fused, n)
        ms_u = timed(unfused, n)
    fused()
    torch.cuda.synchronize()
    from tests.gpu_util import pick_channels
    from oracle import mixer_oracle as O
    chans = pick_channels(Di, 24 if w.seqlen > 8192 else 64, w.seed)
    oout = O.mixer_dtproj_channels(inp, np.arange(Bt), chans, nthreads=0, widen=I.as_f64)
    par = parity_of(w, inp, y, h, cs, chans, oout)
    fb = fwd_bytes(w) - 2 * Bt * L * Di + 2 * Bt * L * R + 2 * Di * R
    peaks = measured_peaks()
    clocks = clk.summary()
    sm_hz = (clocks.get("sm_max_mhz") or 1965.0) * 1e6
    roof = roofline_of("fwd", w, fb, ms_f, peaks, sm_hz, "mamba_mixer_fwd_dtproj")
    roof["traffic"] = None
    return {"metric": "fused conv+selective-scan+gate with dt_proj on the tensor cores: "
                      "algorithmic HBM GB/s", "pass": "dtproj", "unit": "GB/s",
            "value": round(fb / (ms_f * 1e-3) / 1e9, 2), "higher_is_better": True,
            "config": {"workload": w.name, "batch": Bt, "seqlen": L, "d_inner": Di,
                       "d_state": N, "dt_rank": R},
            "fused_ms": round(ms_f, 5), "unfused_ms": round(ms_u, 5),
            "unfused_is": "torch.matmul (cuBLAS bf16) for dt_raw, then mamba_mixer_fwd",
            "algorithmic_bytes_fused": fb, "roofline": roof, "parity": par, "clocks": clocks,
            "gpu_launches": n}


# ----------------------------------------------------------------------------- backward
def bwd_bytes(w: I.Workload) -> int:
    """Algorithmic bytes of one backward: the forward's inputs and dy read once, the fp32
    gradients written once (the tile-state workspace is not counted)."""
    s = w.io_bytes
    Bt, L, Di, N = w.batch, w.seqlen, w.d_inner, w.d_state
    return (4 * Bt * L * Di * s + 2 * Bt * L * N * s + Di * (4 * N + 28)   # x' z dt dy, B C, params
            + 3 * Bt * L * Di * 4 + 2 * Bt * L * N * 4 + Di * (4 * N + 28))  # gradients


def run_bwd(args, w: I.Workload, local_rank: int):
    """--pass bwd: times mamba_mixer_bwd alone (device events, L2 flushed between calls)."""
    import torch
    from selective_state_space_silu_b200 import mixer as M
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M.load_library()
    inp = I.make_inputs(w)
    r = np.random.default_rng(w.seed + 31)
    dy = r.standard_normal((w.batch, w.seqlen, w.d_inner)).astype(np.float32)
    inp["dy"] = I.f32_to_bf16_bits(dy) if w.io_dtype == I.BF16 else dy

    def td(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    d = {k: td(v) for k, v in inp.items()}
    dims = M.make_dims(w.batch, w.seqlen, w.d_inner, w.d_state, 4, M._io_code(d["xp"]))
    ws = torch.empty(max(M.load_library().mamba_mixer_bwd_workspace_bytes(__import__("ctypes").byref(dims)), 16),
                     dtype=torch.uint8, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    fargs = (d["xp"], d["z"], d["dt_raw"], d["B"], d["C"], d["A_log"], d["D"], d["conv_w"],
             d["conv_b"], d["dt_bias"])
    ck = M.new_ckpt(dims, dev)
    y = torch.empty_like(d["xp"])
    fws = M.new_workspace(dims, dev)

    def call():
        M.mamba_mixer_bwd(*fargs, d["dy"], workspace=ws, stream=stream)

    def call_ck():
        M.mamba_mixer_bwd(*fargs, d["dy"], workspace=ws, stream=stream, h_ckpt=ck)

    def fwd_plain():
        M.mamba_mixer_fwd(*fargs, y=y, workspace=fws, stream=stream, want_states=False)

    def fwd_ck():
        M.mamba_mixer_fwd(*fargs, y=y, workspace=fws, stream=stream, want_states=False, h_ckpt=ck)

    def timed(fn, n):
        for _ in range(args.warmup):
            flush.fill_(1.0); torch.sum(flush_rd, dim=0, out=sink)
            fn()
        torch.cuda.synchronize()
        evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(n)]
        for e0, e1 in evs:
            flush.fill_(1.0); torch.sum(flush_rd, dim=0, out=sink)
            e0.record(stream); fn(); e1.record(stream)
        torch.cuda.synchronize()
        return statistics.mean(a.elapsed_time(b) for a, b in evs)

    with ClockSampler(local_rank) as clk:
        ms = timed(call, args.steps)
        ms_fwd = timed(fwd_plain, args.steps)
        ms_fwd_ck = timed(fwd_ck, args.steps)      # also leaves ck for the next one
        ms_ck = timed(call_ck, args.steps)
    nbytes = bwd_bytes(w)
    clocks = clk.summary()
    sm_hz = (clocks.get("sm_max_mhz") or 1965.0) * 1e6
    elems = w.batch * w.seqlen * w.d_inner * w.d_state
    t_floor = 3 * elems / (MUFU_PER_CLK_SM * SMS * sm_hz)   # three exps per element
    peaks = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    return {
        "metric": "mixer backward: achieved algorithmic GB/s", "pass": "backward",
        "value": round(achieved, 2), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "dtype": "bf16" if w.io_dtype == I.BF16 else "f32", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "d_inner": w.d_inner, "d_state": w.d_state,
                   "l2": "flushed between calls", "algorithmic_bytes": nbytes},
        "roofline": {"kernel": "mamba_mixer_bwd", "bound": "alu",
                     "achieved": round(achieved, 2), "peak": round(nbytes / t_floor / 1e9, 2),
                     "unit": "GB/s", "frac": round(t_floor / (ms * 1e-3), 4),
                     "peak_source": "3 exps per (t, d, n) on MUFU (16/clk/SM) x 148 SMs",
                     "hbm_frac": round(achieved / peaks["hbm_gbs"], 4), "traffic": None},
        "checkpointed": {
            "what": "mamba_mixer_fwd_ckpt writes the state before every 16-step tile; "
                    "mamba_mixer_bwd_ckpt reads them instead of recomputing them",
            "bwd_ms": round(ms_ck, 5), "fwd_ckpt_ms": round(ms_fwd_ck, 5),
            "fwd_plain_ms": round(ms_fwd, 5),
            "train_step_ms": round(ms_fwd_ck + ms_ck, 5),
            "train_step_recompute_ms": round(ms_fwd + ms, 5),
            "ckpt_bytes": ck.numel() * 4},
        "gpu_launches": args.steps, "clocks": clocks,
    }


def oracle_sample_bwd(w: I.Workload, target_s: float):
    """The fp64 backward oracle on a bounded sample of the workload: all batch rows, a
    subset of channels, the full sequence (dB/dC then sum over the sample's channels only,
    which costs the same per channel).  Returns (GB/s of backward bytes, cores, description)."""
    from oracle import mixer_oracle as O
    O.build()
    inp = I.make_inputs(w)
    Bt, L, Di = w.batch, w.seqlen, w.d_inner
    dy = np.random.default_rng(w.seed + 31).standard_normal((Bt, L, Di)).astype(np.float32)
    inp["dy"] = I.f32_to_bf16_bits(dy) if w.io_dtype == I.BF16 else dy
    f = I.as_f64

    def run(chans):
        O.mixer_bwd(f(inp["xp"][:, :, chans]), f(inp["z"][:, :, chans]),
                    f(inp["dt_raw"][:, :, chans]), f(inp["B"]), f(inp["C"]), inp["A_log"][chans],
                    inp["D"][chans], inp["conv_w"][chans], inp["conv_b"][chans],
                    inp["dt_bias"][chans], f(inp["dy"][:, :, chans]), nthreads=0)

    probe = np.arange(min(Di, 4))
    t0 = time.perf_counter()
    run(probe)
    dt = max(time.perf_counter() - t0, 1e-4)
    nch = int(min(Di, max(4, len(probe) * target_s / dt)))
    chans = np.linspace(0, Di - 1, nch).astype(np.int64)
    t0 = time.perf_counter()
    run(chans)
    el = time.perf_counter() - t0
    gbs = Bt * L * nch * (bwd_bytes(w) / (Bt * L * Di)) / el / 1e9
    return gbs, O.max_threads(), (f"{w.name} backward: all {Bt} batch rows x {nch} of {Di} channels "
                                  f"x L={L} (fp64 oracle, {el:.2f} s)")


# ----------------------------------------------------------------------------- Mamba2 scan
SSD_Q = 64  # chunk length of the Mamba2 scan kernel


def ssd_bytes(w) -> int:
    """Algorithmic bytes of one Mamba2 scan call: x (and z), dt_raw, B, C read once, y
    written once (bf16), the per-head parameters, h_in read and h_out written (fp32)."""
    Bt, L, H, P, N, G = w.batch, w.seqlen, w.nheads, w.headdim, w.d_state, w.ngroups
    act = Bt * L * H * P * 2
    return (act * (3 if w.gate else 2) + Bt * L * H * 2 + 2 * Bt * L * G * N * 2 + 3 * H * 4
            + Bt * H * P * N * 4 * (2 if w.state else 1))


def ssd_flops(w) -> int:
    """Algorithmic tensor FLOPs of the chunked evaluation with 64-step chunks, causal half
    only: per (row, head, chunk of q steps) q(q+1)/2 (N + P) multiply-adds for C B^T and
    its product with x, plus q N P each for the inter-chunk term and the state update."""
    Bt, L, H, P, N = w.batch, w.seqlen, w.nheads, w.headdim, w.d_state
    total = 0
    full, tail = divmod(L, SSD_Q)
    for q, cnt in ((SSD_Q, full), (tail, 1 if tail else 0)):
        total += cnt * 2 * (q * (q + 1) // 2 * (N + P) + 2 * q * N * P)
    return Bt * H * total


def run_ssd(args, w, local_rank: int):
    """--pass ssd: times mamba2_ssd_fwd alone (device events, L2 flushed between calls);
    for a one-token workload with a cached state, mamba2_ssd_step (the state in place)."""
    import torch
    from selective_state_space_silu_b200 import mixer as M
    from selective_state_space_silu_b200 import ssd as S
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M.load_library()
    inp = I.make_ssd_inputs(w)

    def td(a):
        if a is None:
            return None
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    d = {k: td(v) for k, v in inp.items()}
    y = torch.empty_like(d["x"])
    h_out = torch.empty(w.batch, w.nheads, w.headdim, w.d_state, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_rd = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    sink = torch.empty((), dtype=torch.float32, device=dev)

    step = w.seqlen == 1 and w.state

    def call():
        if step:
            S.mamba2_ssd_step(d["x"], d["dt_raw"], d["A_log"], d["B"], d["C"], d["D"],
                              d["dt_bias"], d["h_in"], z=d["z"], y=y, h_out=d["h_in"],
                              stream=stream)
        else:
            S.mamba2_ssd_fwd(d["x"], d["dt_raw"], d["A_log"], d["B"], d["C"], d["D"],
                             d["dt_bias"], z=d["z"], h_in=d["h_in"], y=y, h_out=h_out,
                             stream=stream)

    for _ in range(args.warmup):
        flush.fill_(1.0); torch.sum(flush_rd, dim=0, out=sink)
        call()
    torch.cuda.synchronize()
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    with ClockSampler(local_rank) as clk:
        for e0, e1 in evs:
            flush.fill_(1.0); torch.sum(flush_rd, dim=0, out=sink)
            e0.record(stream); call(); e1.record(stream)
        torch.cuda.synchronize()
    ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
    nbytes, flops = ssd_bytes(w), (0 if step else ssd_flops(w))  # the step runs no products
    peaks = measured_peaks()
    achieved = nbytes / (ms * 1e-3) / 1e9
    tflops = flops / (ms * 1e-3) / 1e12
    bf16_peak = peaks["bf16_tflops"]
    t_floor = max(nbytes / (peaks["hbm_gbs"] * 1e9), flops / (bf16_peak * 1e12))
    return {
        "metric": ("Mamba2 decode step" if step else "Mamba2 scan (SSD) forward")
                  + ": achieved algorithmic GB/s", "pass": "ssd",
        "value": round(achieved, 2), "unit": "GB/s", "n_gpus": 1, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms, 5), "higher_is_better": True,
        "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "nheads": w.nheads, "headdim": w.headdim, "d_state": w.d_state,
                   "ngroups": w.ngroups, "gate": w.gate, "initial_state": w.state,
                   "chunk": SSD_Q, "l2": "flushed between calls", "algorithmic_bytes": nbytes,
                   "algorithmic_flops": flops},
        "roofline": {"kernel": "ssd_step_kernel" if step else "ssd_fwd_kernel", "bound": "hbm",
                     "achieved": round(achieved, 2),
                     "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": round(achieved / peaks["hbm_gbs"], 4),
                     "peak_source": peak_labels(peaks)[0],
                     "tensor_tflops": None if step else round(tflops, 2),
                     "tensor_frac": None if step else round(tflops / bf16_peak, 4),
                     "tensor_peak_source": peak_labels(peaks)[1],
                     "floor_frac": round(t_floor / (ms * 1e-3), 4),
                     "traffic": recorded_traffic("ssd_step" if step else "ssd", w.name)},
        "gpu_launches": args.steps, "clocks": clk.summary(),
    }


def run_layer(args, w, local_rank: int):
    """--pass layer: the Mamba2 layer's conv + SiLU over x|B|C and its gated RMSNorm, each
    timed alone (device events, L2 flushed between calls) on workload w's shapes."""
    import torch
    from selective_state_space_silu_b200 import mixer as M
    from selective_state_space_silu_b200 import ssd as S
    dev = torch.device("cuda", local_rank)
    torch.cuda.set_device(dev)
    M.load_library()
    Bt, L, H, N, G = w.batch, w.seqlen, w.nheads, w.d_state, w.ngroups
    D, Cc = H * 64, H * 64 + 2 * G * N
    r = np.random.default_rng(w.seed + 7)

    def td(a):
        if a.dtype == np.uint16:
            return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(dev)
        return torch.from_numpy(np.ascontiguousarray(a)).to(dev)

    xbc = td(I.f32_to_bf16_bits(r.standard_normal((Bt, L, Cc), dtype=np.float32)))
    cw = td(r.uniform(-0.5, 0.5, size=(Cc, 4)).astype(np.float32))
    cb = td(r.uniform(-0.5, 0.5, size=Cc).astype(np.float32))
    y = td(I.f32_to_bf16_bits(r.standard_normal((Bt, L, D), dtype=np.float32)))
    z = td(I.f32_to_bf16_bits(r.standard_normal((Bt, L, D), dtype=np.float32)))
    nw = td(r.standard_normal(D).astype(np.float32))
    out = torch.empty_like(y)
    stream = torch.cuda.current_stream(dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    calls = {
        "conv": (lambda: S.mamba2_conv_silu(xbc, cw, cb, nheads=H, ngroups=G, d_state=N,
                                            want_state=False, stream=stream),
                 2 * Bt * L * Cc * 2 + Cc * 20),
        "norm": (lambda: S.mamba2_gated_rmsnorm(y, z, nw, 1e-5, out=out, stream=stream),
                 3 * Bt * L * D * 2 + D * 4),
    }
    peaks = measured_peaks()
    res = {}
    with ClockSampler(local_rank) as clk:
        for name, (fn, nbytes) in calls.items():
            for _ in range(args.warmup):
                flush.fill_(1.0); fn()
            torch.cuda.synchronize()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            for e0, e1 in evs:
                flush.fill_(1.0)
                e0.record(stream); fn(); e1.record(stream)
            torch.cuda.synchronize()
            ms = statistics.mean(a.elapsed_time(b) for a, b in evs)
            gbs = nbytes / (ms * 1e-3) / 1e9
            res[name] = {"ms": round(ms, 5), "GB/s": round(gbs, 2),
                         "frac": round(gbs / peaks["hbm_gbs"], 4), "algorithmic_bytes": nbytes}
    tot_b = sum(v[1] for v in calls.values())
    tot_ms = sum(v["ms"] for v in res.values())
    top = max(res, key=lambda k: res[k]["ms"])
    return {
        "metric": "Mamba2 layer conv + SiLU and gated RMSNorm: achieved algorithmic GB/s",
        "pass": "layer", "value": round(tot_b / (tot_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
        "n_gpus": 1, "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(tot_ms, 5),
        "higher_is_better": True, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "batch": Bt, "seqlen": L, "nheads": H, "d_state": N,
                   "ngroups": G, "channels_conv": Cc, "l2": "flushed between calls"},
        "kernels": res,
        "roofline": {"kernel": "conv_silu_kernel" if top == "conv" else "gated_rmsnorm_kernel",
                     "bound": "hbm", "achieved": res[top]["GB/s"], "peak": peaks["hbm_gbs"],
                     "unit": "GB/s", "frac": res[top]["frac"],
                     "peak_source": peak_labels(peaks)[0], "traffic": None},
        "gpu_launches": 2 * args.steps, "clocks": clk.summary(),
    }


def oracle_sample_ssd(w, target_s: float):
    """The fp64 Mamba2 oracle on a bounded sample: whole sequences of some (row, head)
    pairs.  Returns (GB/s of the workload's bytes per (row, head), cores, description)."""
    from oracle import ssd_oracle as so
    inp = I.make_ssd_inputs(w)
    pairs = [(b, h) for b in range(w.batch) for h in range(w.nheads)]
    t0 = time.perf_counter()
    so.ssd_channels(inp["x"], inp["dt_raw"], inp["A_log"], inp["B"], inp["C"], inp["D"],
                    inp["dt_bias"], pairs[:1], z=inp["z"], h_in=inp["h_in"])
    dt = max(time.perf_counter() - t0, 1e-4)
    n = int(min(len(pairs), max(1, target_s / dt)))
    sel = pairs[:: max(1, len(pairs) // n)][:n]
    t0 = time.perf_counter()
    so.ssd_channels(inp["x"], inp["dt_raw"], inp["A_log"], inp["B"], inp["C"], inp["D"],
                    inp["dt_bias"], sel, z=inp["z"], h_in=inp["h_in"])
    el = time.perf_counter() - t0
    gbs = len(sel) * (ssd_bytes(w) / len(pairs)) / el / 1e9
    return gbs, 1, (f"{w.name}: {len(sel)} of {len(pairs)} (batch row, head) pairs x L={w.seqlen} "
                    f"(fp64 numpy oracle, one thread, {el:.2f} s)")


# ----------------------------------------------------------------------------- oracle
def oracle_sample(w: I.Workload, target_s: float):
    """Times the CPU oracle, as it stands, on a bounded sample of the workload: all batch
    rows, a subset of channels, the full sequence.  Returns (GB/s, cores, description)."""
    from oracle import mixer_oracle as O
    O.build()
    cores = O.max_threads()
    inp = I.make_inputs(w)
    Bt, L, Di = w.batch, w.seqlen, w.d_inner
    per = workload_bytes(w)
    bytes_per_tc = (per["fwd"] + per["step"]) / (Bt * L * Di)
    # size the sample from a quick probe so one pass takes about target_s
    probe = np.arange(min(Di, 8))
    t0 = time.perf_counter()
    O.mixer_channels(inp, np.arange(Bt), probe, widen=I.as_f64, nthreads=0)
    dt = max(time.perf_counter() - t0, 1e-4)
    nch = int(min(Di, max(8, len(probe) * target_s / dt)))
    chans = np.linspace(0, Di - 1, nch).astype(np.int64)
    t0 = time.perf_counter()
    out = O.mixer_channels(inp, np.arange(Bt), chans, widen=I.as_f64, nthreads=0)
    el = time.perf_counter() - t0
    tc = Bt * L * nch
    gbs = tc / el * bytes_per_tc / 1e9
    desc = (f"{w.name}: all {Bt} batch rows x {nch} of {Di} channels x L={L} "
            f"({tc} token-channels, fp64 oracle, {el:.2f} s)")
    return gbs, cores, desc, el, (chans, out)


def run_reference(args, w: I.Workload, rank: int):
    if rank != 0:
        return None
    vals = []
    desc = ""
    cores = 1
    for _ in range(max(1, args.warmup and 1)):
        oracle_sample(w, 1.0)
    for _ in range(args.steps):
        gbs, cores, desc, _, _ = oracle_sample(w, max(2.0, 20.0 / max(args.steps, 1)))
        vals.append(gbs)
    v = statistics.mean(vals)
    return {
        "impl": "reference",
        "metric": METRIC, "value": round(v, 4), "unit": "GB/s", "n_gpus": 1,
        "steps": args.steps, "warmup": args.warmup, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "batch": w.batch, "seqlen": w.seqlen,
                   "d_inner": w.d_inner, "d_state": w.d_state},
        "cpu_baseline": {"value": round(v, 4), "unit": "GB/s", "cores": cores, "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": round(v, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }


# ----------------------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None,
                    help="timed steps (default: 100 for long, 2000 otherwise)")
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long", choices=sorted(I.WORKLOADS))
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the m130 forward and decode step measured beside the default line")
    ap.add_argument("--pass", dest="pass_", choices=["fwd", "bwd", "ssd", "layer", "dtproj"], default="fwd",
                    help="bwd: time the backward (mamba_mixer_bwd) alone on the workload; "
                         "ssd: time the Mamba2 scan (mamba2_ssd_fwd) on --ssd-workload")
    ap.add_argument("--ssd-workload", default="ssd_v3", choices=sorted(I.SSD_WORKLOADS))
    ap.add_argument("--seqlen", type=int, default=None,
                    help="override the workload's sequence length (smaller profiling captures)")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "ours":
        ap.error("--warmup must be >= 3")

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    w = I.WORKLOADS[args.workload]
    if args.steps is None:
        args.steps = 100 if args.workload == "long" else 2000
    if args.seqlen is not None and not w.decode:
        w = w.with_(seqlen=args.seqlen, name=f"{w.name}_L{args.seqlen}")

    if args.impl == "reference":
        res = run_reference(args, w, rank)
        if res is not None:
            print(json.dumps(res), flush=True)
        return

    if args.pass_ != "fwd" and world > 1:
        ap.error("--pass bwd, ssd and layer time one GPU: run them without torchrun")
    if args.pass_ == "layer":
        print(json.dumps(run_layer(args, I.SSD_WORKLOADS[args.ssd_workload], local_rank)), flush=True)
        return
    if args.pass_ == "ssd":
        sw = I.SSD_WORKLOADS[args.ssd_workload]
        if args.seqlen is not None:
            import dataclasses
            sw = dataclasses.replace(sw, seqlen=args.seqlen, name=f"{sw.name}_L{args.seqlen}")
        res = run_ssd(args, sw, local_rank)
        if not args.no_cpu_baseline:
            gbs, cores, desc = oracle_sample_ssd(sw, 10.0)
            res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                   "kind": "oracle", "sample": desc}
        print(json.dumps(res), flush=True)
        return

    if args.pass_ == "dtproj":
        if w.decode or w.io_dtype != I.BF16:
            ap.error("--pass dtproj needs a bf16 forward workload")
        print(json.dumps(run_dtproj(args, w, local_rank)), flush=True)
        return
    if args.pass_ == "bwd":
        if w.decode or w.packed_mean:
            ap.error("--pass bwd needs a plain forward workload")
        res = run_bwd(args, w, local_rank)
        if not args.no_cpu_baseline:
            gbs, cores, desc = oracle_sample_bwd(w, 10.0)
            res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                   "kind": "oracle", "sample": desc}
        print(json.dumps(res), flush=True)
        return

    if world > 1:
        import datetime
        import torch
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        res = run_ours(args, w, rank, world, local_rank)
        if res is not None:
            inp, outs = res.pop("_outs")
            if not args.no_cpu_baseline:
                gbs, cores, desc, _, (chans, oout) = oracle_sample(w, 10.0)
                res["cpu_baseline"] = {"value": round(gbs, 4), "unit": "GB/s", "cores": cores,
                                       "kind": "oracle", "sample": desc}
                if not w.decode:
                    res["parity"] = parity_of(w, inp, *outs, chans, oout)
            if not w.decode and args.no_cpu_baseline:
                from tests.gpu_util import pick_channels
                res["parity"] = parity_of(w, inp, *outs, pick_channels(w.d_inner, 24, w.seed))
            if w.decode:
                from tests.gpu_util import pick_channels
                res["parity"] = parity_of(w, inp, *outs, pick_channels(w.d_inner, 256, w.seed))
            if world == 1 and args.workload == "long" and not args.no_extra:
                import torch
                dev = torch.device("cuda", local_rank)
                peaks = measured_peaks()
                res["m130"] = measure_extra(I.WORKLOADS["m130"], dev, 200, peaks, 96)
                res["decode"] = measure_extra(I.WORKLOADS["decode"], dev, 3000, peaks, 512)
                # the rows beside the forward, timed the same way (their parity is in tests/)
                sub = argparse.Namespace(**{**vars(args), "steps": 20, "warmup": 3})
                bw = run_bwd(sub, I.WORKLOADS["m130"], local_rank)
                res["m130_backward"] = {"ms": bw["ms_per_step"], "gbs": bw["value"],
                                        "roofline": bw["roofline"],
                                        "checkpointed": bw["checkpointed"],
                                        "clocks": bw["clocks"]}
                dp = run_dtproj(sub, I.WORKLOADS["m130"], local_rank)
                res["m130_dtproj"] = {k: dp[k] for k in ("fused_ms", "unfused_ms", "unfused_is",
                                                         "value", "unit", "parity", "clocks")}
                res["m130_dtproj"]["dt_rank"] = dp["config"]["dt_rank"]
            print(json.dumps(res), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()


if __name__ == "__main__":
    main()
