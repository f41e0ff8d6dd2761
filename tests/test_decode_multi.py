"""GPU parity of multi-token decode and of the speculative verify / commit pair
(several new tokens per sequence against resident states: the drafts of the
multi-token-prediction layer, "Qwen3.8 2.4T A95B", key facts and raw config
field mtp_num_hidden_layers), through the C ABI, against the FP64 oracle.

The oracle has no decode of its own for k tokens: decoding k tokens is the
layer run over those k tokens from the resident state and conv window, which
is exactly what oracle.layer computes (the pin "prefill T, then decode = prefill
T + 1" of the oracle tests covers the one-token case).
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


def _oracle(wl, inp, S0, C0, n, m, group=None):
    """The layer over the first m tokens of sequence n from its state and conv window."""
    return oracle.layer(_shape(wl), inp["qkv"][n, :m].cpu(), inp["a"][n, :m].cpu(),
                        inp["b"][n, :m].cpu(), inp["z"][n, :m].cpu(),
                        *[inp[k].cpu() for k in PARAMS], state=S0[n], conv_window=C0[n],
                        group=group)


CASES = [(W.QWEN38_DECODE, 32, 2), (W.QWEN38_DECODE, 16, 4), (W.QWEN38_DECODE, 8, 8),
         (W.QWEN35_DECODE, 16, 3),
         (W.Workload("tiny_decode", 2, 4, 32, dtype="f32", decode_batch=5, state_std=0.02,
                     seed=31), 5, 3)]


@pytest.mark.parametrize("wl,B,k", CASES, ids=lambda x: getattr(x, "name", str(x)))
def test_decode_multi_matches_oracle(cuda_device, wl, B, k):
    cfg = gdn.Config.of(wl)
    inp = W.make_decode(wl, cuda_device, batch=B, tokens=k)
    S0, C0 = inp["state"].cpu(), inp["conv_cache"].cpu()
    y = gdn.decode_multi(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["state"],
                         inp["conv_cache"], *[inp[k_] for k_ in PARAMS])
    torch.cuda.synchronize()
    assert y.shape == (B, k, wl.num_v_heads, wl.head_dim)
    for n in sorted({0, B // 2, B - 1}):
        ref = _oracle(wl, inp, S0, C0, n, k)
        r, m = assert_output_close(y[n], ref["y"], f"y seq {n}")
        rs = assert_state_close(inp["state"][n], ref["state"], f"state seq {n}")
        np.testing.assert_array_equal(to64(inp["conv_cache"][n]), ref["conv_window"])
        report(f"decode_multi {wl.name} k={k} seq {n}", r, m, rs)


@pytest.mark.parametrize("wl,B,k", CASES[:2] + CASES[3:], ids=lambda x: getattr(x, "name", str(x)))
def test_verify_then_commit(cuda_device, wl, B, k):
    """verify leaves the state and conv cache untouched and gives the outputs of all
    k tokens; commit then takes exactly accepted[n] leading tokens of each sequence."""
    cfg = gdn.Config.of(wl)
    inp = W.make_decode(wl, cuda_device, batch=B, tokens=k)
    P = [inp[k_] for k_ in PARAMS]
    S0, C0 = inp["state"].clone(), inp["conv_cache"].clone()
    y_v = gdn.decode_verify(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["state"],
                            inp["conv_cache"], *P)
    torch.cuda.synchronize()
    assert torch.equal(inp["state"], S0) and torch.equal(inp["conv_cache"], C0)
    # the same outputs as the updating decode of all k tokens
    S1, C1 = S0.clone(), C0.clone()
    y_m = gdn.decode_multi(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], S1, C1, *P)
    torch.cuda.synchronize()
    assert torch.equal(y_v, y_m)
    g = torch.Generator().manual_seed(B * 10 + k)
    acc = torch.randint(0, k + 1, (B,), generator=g, dtype=torch.int32)
    acc[0], acc[-1] = 0, k  # none and all accepted
    if B > 2:
        acc[1] = 1
    gdn.decode_commit(cfg, inp["qkv"], inp["a"], inp["b"], inp["state"], inp["conv_cache"],
                      acc.to(cuda_device), *P)
    torch.cuda.synchronize()
    S0c, C0c = S0.cpu(), C0.cpu()
    for n in range(B):
        m = int(acc[n])
        if m == 0:
            assert torch.equal(inp["state"][n], S0[n]) and torch.equal(inp["conv_cache"][n], C0[n])
            continue
        if m == k:  # the same state as the updating decode, to the bit
            assert torch.equal(inp["state"][n], S1[n]) and torch.equal(inp["conv_cache"][n], C1[n])
        if n in (1, B // 2, B - 1):
            ref = _oracle(wl, inp, S0c, C0c, n, m)
            rs = assert_state_close(inp["state"][n], ref["state"], f"state seq {n} m={m}")
            np.testing.assert_array_equal(to64(inp["conv_cache"][n]), ref["conv_window"])
            ry, my = assert_output_close(y_v[n, :m], ref["y"], f"verify y seq {n}")
            report(f"verify/commit {wl.name} k={k} seq {n} m={m}", ry, my, rs)


def test_multi_equals_single_token_decodes_and_prefill(cuda_device):
    """k tokens in one call equal k one-token decodes, and a prefill of the same k
    tokens continuing the sequence (all on the device)."""
    wl = W.QWEN38_DECODE
    cfg = gdn.Config.of(wl)
    B, k = 8, 4
    inp = W.make_decode(wl, cuda_device, batch=B, tokens=k, seed=77)
    P = [inp[k_] for k_ in PARAMS]
    S0, C0 = inp["state"].clone(), inp["conv_cache"].clone()
    S_m, C_m = S0.clone(), C0.clone()
    y_m = gdn.decode_multi(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], S_m, C_m, *P)
    S_s, C_s = S0.clone(), C0.clone()
    ys = []
    for t in range(k):
        ys.append(gdn.decode(cfg, inp["qkv"][:, t].contiguous(), inp["a"][:, t].contiguous(),
                             inp["b"][:, t].contiguous(), inp["z"][:, t].contiguous(), S_s, C_s,
                             *P))
    y_s = torch.stack(ys, 1)
    cu = torch.arange(0, (B + 1) * k, k, dtype=torch.int32, device=cuda_device)
    flat = lambda x: x.reshape(B * k, *x.shape[2:]).contiguous()
    pre = {}
    for algo in ("serial", "chunked"):
        pre[algo] = gdn.prefill(gdn.Config.of(wl, algo), flat(inp["qkv"]), flat(inp["a"]),
                                flat(inp["b"]), flat(inp["z"]), cu, *P, initial_state=S0,
                                initial_conv=C0, return_final_state=True, return_final_conv=True)
    torch.cuda.synchronize()
    assert_output_close(y_m, y_s, "multi vs single-token y", rel=1e-3, mx=1e-2, roundings=2)
    assert_state_close(S_m, S_s, "multi vs single-token state", rel=1e-5)
    assert torch.equal(C_m, C_s)
    # the token-serial prefill runs the same FP32 recurrence: tight agreement
    assert_output_close(flat(y_m), pre["serial"]["y"], "multi vs serial prefill y", rel=1e-3, mx=1e-2,
                        roundings=2)
    assert_state_close(S_m, pre["serial"]["final_state"], "multi vs serial prefill state", rel=1e-5)
    # the chunked prefill (tf32 products) agrees within the stated bounds
    assert_output_close(flat(y_m), pre["chunked"]["y"], "multi vs chunked prefill y", roundings=2)
    assert_state_close(S_m, pre["chunked"]["final_state"], "multi vs chunked prefill state")
    for algo in pre:
        assert torch.equal(C_m, pre[algo]["final_conv"])
