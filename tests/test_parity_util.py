"""The comparison helpers themselves (CPU)."""
import numpy as np
import pytest
import torch

from parity_util import assert_output_close, assert_state_close


def test_bf16_rounding_of_exact_result_passes():
    rng = np.random.default_rng(0)
    ref = rng.standard_normal(10000) * np.exp(rng.standard_normal(10000))  # heavy tail
    got = torch.tensor(ref, dtype=torch.float32).to(torch.bfloat16)  # correctly rounded
    assert_output_close(got, ref)


def test_real_errors_fail():
    rng = np.random.default_rng(1)
    ref = rng.standard_normal(10000)
    bad = ref.copy()
    bad[17] += 0.2  # one element off by 0.2 rms
    with pytest.raises(AssertionError, match="max abs"):
        assert_output_close(torch.tensor(bad, dtype=torch.float32), ref)
    with pytest.raises(AssertionError, match="rel L2"):
        assert_output_close(torch.tensor(ref * 1.02, dtype=torch.float32), ref)
    with pytest.raises(AssertionError, match="rel L2"):
        assert_state_close(torch.tensor(ref * 0.98), ref)
    with pytest.raises(AssertionError, match="non-finite"):
        x = torch.tensor(ref, dtype=torch.float32)
        x[3] = float("nan")
        assert_output_close(x, ref)
