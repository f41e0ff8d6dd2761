"""GPU parity of the chunked prefill's sequence split and of long single sequences.

The state map of a stretch of tokens is affine in the state entering it,
S_end = S0 M + R.  With gdn_config.segments = P the library computes (M, R)
of every segment but the last, chains them into each segment's entering
state and then scans all segments in parallel.  These tests compare that
against the oracle's token-by-token recurrence over whole sequences:
  - under gates that carry the state across segments (almost no decay, beta
    about 0.12), where a wrong M, R or chain shows at the start of every
    segment and in the final state;
  - with more segments than some sequences have chunks (empty segments);
  - on one 262,144-token sequence (the Qwen3.8 context window) at the Qwen3.8
    and Qwen3.5-397B layer shapes, with the library's own choice of segments.
"""
import numpy as np
import pytest
import torch

import linear_attention_layer_causal_b200 as gdn
import oracle
from linear_attention_layer_causal_b200 import workloads as W
from parity_util import assert_output_close, assert_state_close, report, to64

pytestmark = pytest.mark.gpu

PARAMS = ("conv_w", "A_log", "dt_bias", "norm_w")


def _shape(wl):
    return oracle.Shape(wl.num_qk_heads, wl.num_v_heads, wl.head_dim, wl.conv_kernel)


def _prefill(cfg, inp, **kw):
    return gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"],
                       *[inp[k] for k in PARAMS], initial_state=inp.get("initial_state"),
                       check_status=True, **kw)


def _oracle_seq(wl, inp, n, group, heads=None):
    cu = inp["cu_seqlens"].tolist()
    s, e = cu[n], cu[n + 1]
    S0 = inp.get("initial_state")
    return oracle.layer(_shape(wl), inp["qkv"][s:e], inp["a"][s:e], inp["b"][s:e],
                        inp["z"][s:e], *[inp[k] for k in PARAMS],
                        state=None if S0 is None else S0[n], group=group, heads=heads)


def _segments_used(cfg, batch, N):
    """The P a call runs with, as the library reports it and as its workspace shows."""
    P = gdn.prefill_segments(cfg, batch, N)
    base = gdn.prefill_workspace_size(gdn.Config(**{**cfg.__dict__, "segments": 1}), batch, N)
    per = 3 * batch * cfg.num_v_heads * cfg.head_dim ** 2 * 4
    assert gdn.prefill_workspace_size(cfg, batch, N) - base == (P - 1) * per
    return P


@pytest.mark.parametrize("segments", [2, 3, 5, 16])
def test_split_matches_oracle(cuda_device, segments):
    """Varlen Qwen3.5-shape prefill with a slowly forgetting state, split P ways."""
    wl = W.SPLIT_MEMORY
    cfg = gdn.Config.of(wl, "chunked", segments)
    inp = W.make_prefill(wl, cuda_device)
    N, B = int(inp["cu_seqlens"][-1]), len(inp["seqlens"])
    assert _segments_used(cfg, B, N) == segments
    out = _prefill(cfg, inp, return_final_state=True, return_final_conv=True, return_o_raw=True)
    one = _prefill(gdn.Config.of(wl, "chunked", 1), inp, return_final_state=True,
                   return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    G = wl.num_v_heads // wl.num_qk_heads
    for n, group in [(0, 3), (1, 7), (2, 10), (3, 0), (4, 15)]:
        heads = list(range(group * G, (group + 1) * G))
        ref = _oracle_seq(wl, inp, n, group)
        s, e = cu[n], cu[n + 1]
        r = m = None
        if e > s:
            r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n} group {group}")
            assert_output_close(out["o_raw"][s:e, heads], ref["o"], f"o seq {n} group {group}")
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"split P={segments} seq {n} len {e - s} group {group}", r, m, rs)
    # the split and the single chain: the same outputs and states up to rounding
    r, _ = assert_output_close(out["o_raw"], one["o_raw"], "split vs unsplit o")
    rs = assert_state_close(out["final_state"], one["final_state"], "split vs unsplit state")
    report(f"split P={segments} vs P=1 (all heads)", r, None, rs)
    for n in range(B):
        s, e = cu[n], cu[n + 1]
        hist = torch.cat([torch.zeros_like(inp["qkv"][:3]), inp["qkv"][s:e]])
        assert torch.equal(out["final_conv"][n], hist[-3:])


def test_split_state_only_and_no_initial_state(cuda_device):
    """No initial state and no outputs but y: the split's chain starts from zero."""
    wl = W.SPLIT_MEMORY
    inp = W.make_prefill(wl, cuda_device, seqlens=(3000,), seed=77)
    inp["initial_state"] = None
    out = _prefill(gdn.Config.of(wl, "chunked", 6), inp, return_final_state=True)
    torch.cuda.synchronize()
    G = wl.num_v_heads // wl.num_qk_heads
    group = 6
    heads = list(range(group * G, (group + 1) * G))
    ref = _oracle_seq(wl, inp, 0, group)
    r, m = assert_output_close(out["y"][:, heads], ref["y"], "y")
    rs = assert_state_close(out["final_state"][0, heads], ref["state"], "state")
    report("split P=6 zero initial state", r, m, rs)


@pytest.mark.parametrize("wl", [W.QWEN38_262K, W.QWEN35_262K], ids=lambda w: w.name)
def test_262k_single_sequence(cuda_device, wl):
    """One 262,144-token sequence: the library's segments; two value heads against the oracle."""
    cfg = gdn.Config.of(wl)
    inp = W.make_prefill(wl, cuda_device)
    N = int(inp["cu_seqlens"][-1])
    P = _segments_used(cfg, 1, N)
    # 128 value heads fill the SMs with one chain each; 64 leave room for a split
    assert (P == 1) if wl.num_v_heads == 128 else (P >= 2)
    out = _prefill(cfg, inp, return_final_state=True, return_final_conv=True)
    torch.cuda.synchronize()
    G = wl.num_v_heads // wl.num_qk_heads
    group = 5
    heads = [group * G, group * G + G - 1]
    ref = _oracle_seq(wl, inp, 0, group, heads)
    r, m = assert_output_close(out["y"][:, heads], ref["y"], "y")
    rs = assert_state_close(out["final_state"][0, heads], ref["state"], "state")
    report(f"{wl.name} (P={P}) heads {heads}", r, m, rs)
    # whole-tensor properties: finite outputs everywhere, the exact conv window
    for t0 in range(0, N, 32768):
        assert torch.isfinite(out["y"][t0:t0 + 32768].float()).all()
    np.testing.assert_array_equal(to64(out["final_conv"][0]), to64(inp["qkv"][N - 3:N]))


@pytest.mark.parametrize("segments", [3, 7])
def test_split_float32_activations(cuda_device, segments):
    """fp32 activations: the passes read the front end's convolved v by TMA
    instead of convolving it; all heads of a small layer against the oracle."""
    wl = W.Workload("split_f32", 2, 4, 128, dtype="f32", seqlens=(700, 0, 300), state_std=0.02,
                    seed=13, gates="long_memory:-8:-2")
    cfg = gdn.Config.of(wl, "chunked", segments)
    inp = W.make_prefill(wl, cuda_device)
    out = _prefill(cfg, inp, return_final_state=True, return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(cu) - 1):
        s, e = cu[n], cu[n + 1]
        ref = oracle.prefill(_shape(wl), inp["qkv"][s:e], inp["a"][s:e], inp["b"][s:e], inp["z"][s:e],
                             [0, e - s], *[inp[k] for k in PARAMS],
                             initial_state=inp["initial_state"][n:n + 1])
        r = m = None
        if e > s:
            r, m = assert_output_close(out["y"][s:e], ref["y"], f"y seq {n}")
            assert_output_close(out["o_raw"][s:e], ref["o"], f"o seq {n}")
        rs = assert_state_close(out["final_state"][n], ref["state"][0], f"state seq {n}")
        report(f"split fp32 P={segments} seq {n} len {e - s}", r, m, rs)
