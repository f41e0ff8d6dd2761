"""Comparison helpers for GPU-vs-oracle parity.

Tolerances against the FP64 oracle: output relative L2 <= 1e-2, max abs
error <= 5e-2 * rms(oracle output), final-state relative L2 <= 1e-2.

The max-abs bound applies to the computed value before its final rounding
to the output's storage format: a bf16 output element is the correctly
computed value rounded to 8 significant bits, which alone moves it by up to
the unit roundoff of that format, 2^-8 |y|, and |y| reaches ~60 rms(y) in
these workloads.  So for a bf16 output each element may additionally differ
by that unit roundoff of the reference value (2^-8 |y_ref|); float32 outputs
(o_raw, states) get no such allowance.

report() prints, for each comparison, how much of the budget it used (the
relative L2 over 1e-2, the max-abs excess over 5e-2 rms), so that a drift
toward a bound shows long before it fails; with GDN_PARITY_REPORT set the
same lines are appended to that file.
"""
import os

import numpy as np

OUT_REL_L2 = 1e-2
OUT_MAX_ABS_RMS = 5e-2
STATE_REL_L2 = 1e-2


def to64(x):
    if hasattr(x, "detach"):
        return x.detach().to("cpu").double().numpy()
    return np.asarray(x, dtype=np.float64)


def rel_l2(got, ref):
    got, ref = to64(got), to64(ref)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((got - ref).ravel()) / (den if den > 0 else 1.0))


def max_abs_over_rms(got, ref):
    got, ref = to64(got), to64(ref)
    rms = float(np.sqrt(np.mean(ref ** 2))) if ref.size else 0.0
    return float(np.max(np.abs(got - ref))) / (rms if rms > 0 else 1.0) if ref.size else 0.0


def format_ulp(got):
    """Relative size of one unit in the last place of the storage format of `got`."""
    dt = str(getattr(got, "dtype", "float64"))
    return 2.0 ** -8 if "bfloat16" in dt else (2.0 ** -23 if "float32" in dt else 0.0)


def assert_output_close(got, ref, what="y", rel=OUT_REL_L2, mx=OUT_MAX_ABS_RMS, roundings=1):
    """`roundings`: how many roundings to the output format separate got from ref (1
    against the oracle; 2 when both sides are outputs of the library, each rounded)."""
    ulp = roundings * format_ulp(got)
    g, rf = to64(got), to64(ref)
    assert np.all(np.isfinite(g)), f"{what}: non-finite values"
    r = rel_l2(g, rf)
    assert r <= rel, f"{what}: rel L2 {r:.3e} > {rel:.1e}"
    if rf.size == 0:
        return r, 0.0
    rms = float(np.sqrt(np.mean(rf ** 2))) or 1.0
    excess = np.abs(g - rf) - ulp * np.abs(rf)  # error beyond the output format's own rounding
    m = float(np.max(excess)) / rms
    assert m <= mx, f"{what}: max abs (beyond format rounding) / rms {m:.3e} > {mx:.1e}"
    return r, m


def assert_state_close(got, ref, what="state", rel=STATE_REL_L2):
    r = rel_l2(got, ref)
    assert np.all(np.isfinite(to64(got))), f"{what}: non-finite values"
    assert r <= rel, f"{what}: rel L2 {r:.3e} > {rel:.1e}"
    return r


def report(name, rel=None, maxabs=None, state_rel=None):
    """One line of budget use: each figure as a fraction of its tolerance bound."""
    parts = [name]
    if rel is not None:
        parts.append(f"y_rel={rel:.3e} ({rel / OUT_REL_L2:.1%} of bound)")
    if maxabs is not None:
        parts.append(f"y_maxabs_excess={maxabs:.3e}rms ({maxabs / OUT_MAX_ABS_RMS:.1%} of bound)")
    if state_rel is not None:
        parts.append(f"state_rel={state_rel:.3e} ({state_rel / STATE_REL_L2:.1%} of bound)")
    line = "PARITY " + " ".join(parts)
    print(line)
    path = os.environ.get("GDN_PARITY_REPORT")
    if path:
        with open(path, "a") as f:
            f.write(line + "\n")
