"""Sealed tolerance classes for comparing the CUDA path with the fp64 oracle.

fp32 I/O: abs(a-b) <= 1e-5 + 1e-3*max(|a|,|b|) -- the agreement test of the openfluke
"Apple Mamba stress test" (section "What the results mean", within_tolerance_pct).

bf16 I/O with fp32 state: abs(a-b) <= 1e-3 + 2e-2*max(|a|,|b|).  The 2e-2 relative
bound is the stated bf16 bound for this operator; the 1e-3 absolute floor covers outputs
near zero, where a pure relative bound cannot hold for values rounded to bf16 (one bf16
ulp at 0.06 is 2.4e-4, and the gate multiplies by SiLU(z) of order 1).

Non-finite values never count as a match, on either side (the stress test reports
non-finite values as errors, never as matches).  Tests that feed non-finite inputs on
purpose check where they propagate with `same_nonfinite_pattern`, separately, and compare
only the finite part with the class.
Tolerances are sealed: a failing comparison is a finding, not a reason to widen them.
"""

import numpy as np

TOL = {
    "f32": (1e-5, 1e-3),
    "bf16": (1e-3, 2e-2),
}


def within(a, b, io_dtype):
    """Elementwise mask of the tolerance test (a: device result, b: oracle)."""
    atol, rtol = TOL[io_dtype]
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    fin = np.isfinite(a) & np.isfinite(b)
    ok = np.zeros(a.shape, dtype=bool)
    ok[fin] = np.abs(a[fin] - b[fin]) <= atol + rtol * np.maximum(np.abs(a[fin]), np.abs(b[fin]))
    return ok


def same_nonfinite_pattern(a, b, what=""):
    """NaN-propagation check, kept apart from the tolerance class: the device result and the
    oracle must be non-finite at exactly the same positions, with NaN where the oracle has
    NaN and the same infinity where it has one.  Returns the mask of positions that are
    finite on both sides (the part the tolerance class then judges)."""
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    np.testing.assert_array_equal(np.isnan(a), np.isnan(b), err_msg=f"{what}: NaN positions")
    inf_b = np.isinf(b)
    np.testing.assert_array_equal(np.isinf(a), inf_b, err_msg=f"{what}: infinite positions")
    np.testing.assert_array_equal(a[inf_b], b[inf_b], err_msg=f"{what}: signs of infinities")
    return np.isfinite(a) & np.isfinite(b)


def report(a, b, io_dtype):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    ok = within(a, b, io_dtype)
    d = np.abs(a - b)
    with np.errstate(invalid="ignore", divide="ignore"):
        rel = d / np.maximum(np.abs(b), 1e-30)
    return {
        "n": int(a.size),
        "within_pct": 100.0 * float(ok.mean()) if a.size else 100.0,
        "exact_pct": 100.0 * float((a == b).mean()) if a.size else 100.0,
        "max_abs": float(np.nanmax(d)) if a.size else 0.0,
        "max_rel": float(np.nanmax(rel)) if a.size else 0.0,
        "worst": None if ok.all() else int(np.argmin(ok.reshape(-1))),
    }


def assert_close(a, b, io_dtype, what=""):
    r = report(a, b, io_dtype)
    if r["within_pct"] < 100.0:
        idx = np.unravel_index(r["worst"], np.shape(a))
        raise AssertionError(
            f"{what}: {100 - r['within_pct']:.4f}% outside {io_dtype} tolerance "
            f"(max_abs {r['max_abs']:.3e}, max_rel {r['max_rel']:.3e}); first at {idx}: "
            f"got {np.asarray(a)[idx]!r}, oracle {np.asarray(b)[idx]!r}")
    return r


def within_grad(a, b, io_dtype):
    """Tolerance for gradients (device fp32 vs fp64 oracle): the class's bound plus a floor
    of rtol times the RMS of the oracle tensor.  Most gradients are sums of many terms of
    both signs (over time, channels or batch rows), whose rounding error scales with the
    size of the terms rather than with the possibly cancelled result; the tensor's RMS
    stands in for that size.  Same classes: fp32 I/O (precise math) and bf16 I/O (MUFU)."""
    atol, rtol = TOL[io_dtype]
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    rms = float(np.sqrt(np.mean(b[np.isfinite(b)] ** 2))) if b.size else 0.0
    fin = np.isfinite(a) & np.isfinite(b)
    ok = np.zeros(a.shape, dtype=bool)
    ok[fin] = np.abs(a[fin] - b[fin]) <= (atol + rtol * rms +
                                          rtol * np.maximum(np.abs(a[fin]), np.abs(b[fin])))
    return ok


def assert_close_grad(a, b, io_dtype, what=""):
    ok = within_grad(a, b, io_dtype)
    if not ok.all():
        a = np.asarray(a, dtype=np.float64)
        b = np.asarray(b, dtype=np.float64)
        idx = np.unravel_index(int(np.argmin(ok.reshape(-1))), a.shape)
        d = np.abs(a - b)
        raise AssertionError(
            f"{what}: {100 * (1 - ok.mean()):.4f}% outside the {io_dtype} gradient tolerance "
            f"(max_abs {np.nanmax(d):.3e}, oracle rms {np.sqrt(np.mean(b ** 2)):.3e}); first at "
            f"{idx}: got {a[idx]!r}, oracle {b[idx]!r}")


def assert_close_tc(a, b, what=""):
    """Tolerance for the Mamba2 scan's tensor-core path (bf16 operands, fp32 sums) against
    the fp64 oracle: abs(a-b) <= 1e-3 + 2e-2*max(|a|,|b|) + 2e-2*RMS(oracle tensor).

    Derivation: besides the bf16 output rounding (the 2e-2 relative term), each output
    is a sum of many products whose operands include values rounded once to bf16 (relative
    error at most 2^-9, about 1.1e-3 RMS for round-to-nearest): the masked C B^T entries,
    the carried state used for the inter-chunk term, and the Delta-weighted x of the state
    update.  The error of such a sum is about 2^-9/sqrt(3) times the root of the summed
    squares of its terms, which for terms of both signs is of the order of the output's
    RMS: about 1.1e-3 RMS per rounded operand set, under 6e-3 RMS at five standard
    deviations for the two sets that meet in one output.  2e-2 RMS leaves a factor of 3 over that."""
    assert_close_grad(a, b, "bf16", what)
