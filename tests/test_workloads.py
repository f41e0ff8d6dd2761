"""The seeded input generators against the recipe they state: shapes, dtypes,
determinism, and the distributions of every draw (CPU)."""
import math

import pytest
import torch

from linear_attention_layer_causal_b200 import workloads as W

# wide enough in heads that the per-head draws (A_log, dt_bias) have
# thousands of samples, short enough in tokens to stay small
STATS = W.Workload("stats", 64, 4096, 32, seqlens=(3, 0, 5), state_std=0.02, state_every=2, seed=4)


def _std(x):
    return x.double().std().item()


def _mean(x):
    return x.double().mean().item()


def test_prefill_shapes_dtypes_and_offsets():
    for wl in (W.TINY, STATS, W.Workload("b", 2, 4, 128, seqlens=(7, 1, 0, 9), seed=2)):
        inp = W.make_prefill(wl)
        lens = list(wl.seqlens)
        N, B, H, d = sum(lens), len(lens), wl.num_v_heads, wl.head_dim
        assert inp["seqlens"] == lens
        assert inp["cu_seqlens"].dtype == torch.int32
        assert inp["cu_seqlens"].tolist() == [sum(lens[:i]) for i in range(B + 1)]
        assert inp["qkv"].shape == (N, wl.conv_dim) and inp["qkv"].dtype == wl.torch_dtype
        assert inp["a"].shape == inp["b"].shape == (N, H)
        assert inp["z"].shape == (N, H, d) and inp["z"].dtype == wl.torch_dtype
        assert inp["conv_w"].shape == (wl.conv_dim, 4) and inp["conv_w"].dtype == torch.float32
        assert inp["A_log"].shape == inp["dt_bias"].shape == (H,)
        assert inp["norm_w"].shape == (d,)
        if wl.state_std > 0:
            assert inp["initial_state"].shape == (B, H, d, d)
        else:
            assert inp["initial_state"] is None


def test_same_seed_same_bytes_other_seed_other_bytes():
    a, b = W.make_prefill(STATS), W.make_prefill(STATS)
    for k in ("qkv", "a", "b", "z", "conv_w", "A_log", "dt_bias", "norm_w", "initial_state"):
        assert torch.equal(a[k], b[k]), k
    c = W.make_prefill(STATS, seed=5)
    assert not torch.equal(a["qkv"], c["qkv"])
    # lengths given by the caller replace the workload's
    d = W.make_prefill(STATS, seqlens=(8,))
    assert d["qkv"].shape[0] == 8 and d["cu_seqlens"].tolist() == [0, 8]


def test_default_draws_follow_the_stated_distributions():
    inp = W.make_prefill(STATS)
    for k in ("qkv", "a", "b", "z"):  # N(0, 1), cast to the activation dtype
        x = inp[k].float()
        assert abs(_mean(x)) < 0.02 and abs(_std(x) - 1.0) < 0.02, k
    assert abs(_mean(inp["conv_w"])) < 0.01 and abs(_std(inp["conv_w"]) - 0.5) < 0.01
    eA = inp["A_log"].exp()  # U(1, 16): mean 8.5, std 15 / sqrt(12)
    assert eA.min().item() >= 1.0 - 1e-6 and eA.max().item() <= 16.0 + 1e-5
    assert abs(_mean(eA) - 8.5) < 0.3 and abs(_std(eA) - 15 / math.sqrt(12)) < 0.2
    assert abs(_mean(inp["dt_bias"])) < 0.04 and abs(_std(inp["dt_bias"]) - 0.5) < 0.03
    w = inp["norm_w"]  # 1 + 0.1 N(0, 1), 32 samples
    assert (w - 1).abs().max().item() < 0.5 and 0.04 < _std(w) < 0.17
    S = inp["initial_state"]  # N(0, 0.02^2) for sequences 0, 2; zero for 1
    assert torch.count_nonzero(S[1]) == 0
    assert abs(_std(S[0]) - 0.02) < 0.001 and abs(_std(S[2]) - 0.02) < 0.001


@pytest.mark.parametrize("spec,dt_bias,b_mean", [("long_memory:-4", -4.0, 2.0),
                                                 ("long_memory:-8:-2", -8.0, -2.0)])
def test_long_memory_gates(spec, dt_bias, b_mean):
    wl = W.Workload("lm", 16, 64, 32, seqlens=(256,), seed=9, gates=spec)
    inp = W.make_prefill(wl)
    assert torch.count_nonzero(inp["A_log"]) == 0
    assert torch.all(inp["dt_bias"] == dt_bias)
    b = inp["b"].float()
    assert abs(_mean(b) - b_mean) < 0.02 and abs(_std(b) - 0.5) < 0.02
    # a keeps the N(0, 1) draw, so g = -softplus(a + dt_bias) is small
    g = -torch.nn.functional.softplus(inp["a"].double() + dt_bias)
    assert g.mean().item() > -0.05


def test_varlen_lengths_are_seeded_integers_in_range():
    wl = W.QWEN36_VARLEN
    count, lo, hi = wl.varlen
    lens = W.seqlens_of(wl)
    assert len(lens) == count and all(lo <= n <= hi for n in lens)
    assert lens == W.seqlens_of(wl)
    assert len(set(lens)) > count // 2


def test_decode_shapes_single_and_multi_token():
    wl = W.Workload("dec", 2, 4, 32, decode_batch=3, state_std=0.02, seed=6)
    one = W.make_decode(wl)
    assert one["qkv"].shape == (3, wl.conv_dim) and one["z"].shape == (3, 4, 32)
    assert one["state"].shape == (3, 4, 32, 32) and one["conv_cache"].shape == (3, 3, wl.conv_dim)
    k = W.make_decode(wl, tokens=5)
    assert k["qkv"].shape == (3, 5, wl.conv_dim) and k["a"].shape == (3, 5, 4)
    assert k["z"].shape == (3, 5, 4, 32)
    assert torch.equal(one["qkv"], W.make_decode(wl)["qkv"])


def test_kda_shapes_and_draws():
    wl = W.Workload("kda", 8, 8, 32, seqlens=(40, 0, 9), state_std=0.02, seed=3)
    inp = W.make_kda_prefill(wl)
    N, H, d = 49, 8, 32
    assert inp["qkv"].shape == (N, 3 * H * d)
    assert inp["zdec"].shape == inp["gate"].shape == (N, H, d) and inp["b"].shape == (N, H)
    assert inp["conv_w"].shape == (3 * H * d, 4) and inp["A_log"].shape == (H,)
    assert inp["initial_state"].shape == (3, H, d, d)
    eA = inp["A_log"].exp()
    assert eA.min().item() >= 1.0 - 1e-6 and eA.max().item() <= 16.0 + 1e-5
    dec = W.make_kda_decode(wl, batch=2)
    assert dec["state"].shape == (2, H, d, d) and dec["conv_cache"].shape == (2, 3, 3 * H * d)
