"""Comparison helpers for GPU-vs-oracle parity.

Tolerances (bf16 operands, FP32 accumulation and state, against the FP64
oracle): output relative L2 <= 1e-2, max abs error <= 5e-2 * rms(oracle
output), final-state relative L2 <= 1e-2.
"""
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


def assert_output_close(got, ref, what="y", rel=OUT_REL_L2, mx=OUT_MAX_ABS_RMS):
    r, m = rel_l2(got, ref), max_abs_over_rms(got, ref)
    assert np.all(np.isfinite(to64(got))), f"{what}: non-finite values"
    assert r <= rel, f"{what}: rel L2 {r:.3e} > {rel:.1e}"
    assert m <= mx, f"{what}: max abs / rms {m:.3e} > {mx:.1e}"
    return r, m


def assert_state_close(got, ref, what="state", rel=STATE_REL_L2):
    r = rel_l2(got, ref)
    assert np.all(np.isfinite(to64(got))), f"{what}: non-finite values"
    assert r <= rel, f"{what}: rel L2 {r:.3e} > {rel:.1e}"
    return r
