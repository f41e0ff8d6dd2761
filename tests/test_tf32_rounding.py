"""The float32 -> tf32 rounding used for the tensor-core operands (round to
nearest, ties away from zero) is written on the bit pattern as
(bits + 0x1000) & 0xffffe000.  This checks that expression against the
definition: the nearer of the two tf32 neighbours of x (10 explicit mantissa
bits), ties to the larger magnitude, computed with exact float64 arithmetic."""
import numpy as np
import pytest


def bit_rule(x32):
    b = x32.view(np.uint32).astype(np.uint64)
    return (((b + 0x1000) & 0xFFFFE000) & 0xFFFFFFFF).astype(np.uint32).view(np.float32)


def nearest_tf32(x32):
    """The definition, value by value: candidates are x truncated to tf32 and the
    next tf32 away from zero; float64 holds both and the differences exactly."""
    out = np.empty_like(x32)
    for i, x in enumerate(x32):
        b = int(np.float32(x).view(np.uint32))
        lo = np.uint32(b & 0xFFFFE000).view(np.float32)            # toward zero
        hi_bits = (b & 0xFFFFE000) + 0x2000                        # next tf32 away from zero
        hi = np.uint32(hi_bits & 0xFFFFFFFF).view(np.float32) if hi_bits < 2**32 else lo
        dx_lo = abs(float(x) - float(lo))
        dx_hi = abs(float(hi) - float(x)) if np.isfinite(hi) else np.inf
        out[i] = hi if dx_hi <= dx_lo else lo                       # tie -> larger magnitude
        if not np.isfinite(hi) and dx_lo >= 2.0 ** (np.frexp(float(lo))[1] - 12):
            out[i] = hi                                             # rounds past the largest tf32
    return out


@pytest.mark.parametrize("seed", [0, 1])
def test_bit_rule_is_nearest_ties_away(seed):
    rng = np.random.default_rng(seed)
    x = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(5000) * 1e-30).astype(np.float32),   # tiny and subnormal
        (rng.standard_normal(5000) * 1e30).astype(np.float32),    # large
    ])
    # exact ties (low 13 bits = 0x1000) and near-ties, both signs, and carries
    # into the exponent (mantissa all ones in the kept bits)
    base = rng.integers(0, 2**31 - 2**24, 4000, dtype=np.uint64) & ~np.uint64(0x1FFF)
    ties = (base | 0x1000).astype(np.uint32)
    below = (base | 0x0FFF).astype(np.uint32)
    carry = ((base & ~np.uint64(0x7FFFFF)) | 0x7FF000).astype(np.uint32)
    special = np.concatenate([ties, below, carry]).view(np.float32)
    x = np.concatenate([x, special, -special])
    x = x[np.isfinite(x)]
    got = bit_rule(x)
    want = nearest_tf32(x)
    assert np.array_equal(got.view(np.uint32), want.view(np.uint32))
    assert np.all(got.view(np.uint32) & 0x1FFF == 0)
