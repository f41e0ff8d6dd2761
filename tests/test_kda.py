"""GPU parity of Kimi Delta Attention (the per-channel-decay variant, "Inkling vs
Kimi K3", component table, linear-attention and output-gate rows) through the
C ABI, against the FP64 oracle's KDA stages (which tests/test_oracle_kda_pins.py
pins to the Gated DeltaNet rule, the matrix form of the update and closed forms).
"""
import numpy as np
import pytest
import torch

import linear_attention_layer_causal_b200 as gdn
import oracle
from linear_attention_layer_causal_b200 import workloads as W
from parity_util import assert_output_close, assert_state_close, report, to64

pytestmark = pytest.mark.gpu

PK = ("conv_w", "A_log", "norm_w")


def _shape(wl):
    return oracle.Shape(wl.num_qk_heads, wl.num_v_heads, wl.head_dim, wl.conv_kernel)


@pytest.mark.parametrize("wl", [
    W.KIMI_K3_KDA,
    W.Workload("kda_small", 4, 4, 32, dtype="f32", seqlens=(0, 1, 5, 70, 33), state_std=0.02, seed=7),
    W.Workload("kda_edge", 2, 2, 128, seqlens=(3, 0, 129, 64), state_std=0.02, seed=8),
], ids=lambda w: w.name)
def test_kda_prefill_matches_oracle(cuda_device, wl):
    cfg = gdn.Config.of(wl)
    inp = W.make_kda_prefill(wl, cuda_device)
    B = len(inp["seqlens"])
    g = torch.Generator(device=cuda_device).manual_seed(3)
    conv = torch.randn((B, 3, wl.conv_dim), generator=g, device=cuda_device).to(wl.torch_dtype)
    out = gdn.kda_prefill(cfg, inp["qkv"], inp["zdec"], inp["b"], inp["gate"], inp["cu_seqlens"],
                          *[inp[k] for k in PK], initial_state=inp["initial_state"],
                          initial_conv=conv, return_final_state=True, return_final_conv=True,
                          return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    heads = list(range(wl.num_v_heads)) if wl.num_v_heads <= 8 else [0, 37, 95]
    for n in range(B):
        s, e = cu[n], cu[n + 1]
        ref = oracle.kda_layer(_shape(wl), inp["qkv"][s:e], inp["zdec"][s:e], inp["b"][s:e],
                               inp["gate"][s:e], *[inp[k] for k in PK],
                               state=inp["initial_state"][n], conv_window=conv[n], heads=heads)
        if e > s:
            r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n}")
            assert_output_close(out["o_raw"][s:e, heads], ref["o"], f"o seq {n}")
        else:
            r = m = None
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"kda {wl.name} seq {n} len {e - s}", r, m, rs)
    # the final conv window: the last 3 pre-conv rows of [window; sequence]
    for n in range(B):
        s, e = cu[n], cu[n + 1]
        hist = torch.cat([conv[n], inp["qkv"][s:e]])
        assert torch.equal(out["final_conv"][n], hist[-3:])


def test_kda_decode_matches_oracle_and_continues_prefill(cuda_device):
    """Decode against the oracle, and prefill(T) + decode(1) = prefill(T + 1) on the device."""
    wl = W.KIMI_K3_KDA
    cfg = gdn.Config.of(wl)
    d = W.make_kda_decode(wl, cuda_device, batch=6)
    S0, C0 = d["state"].cpu(), d["conv_cache"].cpu()
    y = gdn.kda_decode(cfg, d["qkv"], d["zdec"], d["b"], d["gate"], d["state"], d["conv_cache"],
                       *[d[k] for k in PK])
    torch.cuda.synchronize()
    heads = [1, 50, 94]
    for n in (0, 5):
        ref = oracle.kda_layer(_shape(wl), d["qkv"][n:n + 1], d["zdec"][n:n + 1], d["b"][n:n + 1],
                               d["gate"][n:n + 1], *[d[k] for k in PK], state=S0[n],
                               conv_window=C0[n], heads=heads)
        r, m = assert_output_close(y[n:n + 1, heads], ref["y"], f"decode y seq {n}")
        rs = assert_state_close(d["state"][n, heads], ref["state"], f"decode state seq {n}")
        D, H = wl.head_dim, wl.num_v_heads
        cols = [part * H * D + h * D + i for part in range(3) for h in heads for i in range(D)]
        np.testing.assert_array_equal(to64(d["conv_cache"][n][:, cols]), ref["conv_window"])
        # every channel's window shifts by the decoded row
        assert torch.equal(d["conv_cache"][n].cpu(), torch.cat([C0[n], d["qkv"][n:n + 1].cpu()])[-3:])
        report(f"kda decode seq {n}", r, m, rs)
    # continuation on the device
    T = 200
    inp = W.make_kda_prefill(wl, cuda_device, seqlens=(T + 1,), seed=33)
    P = [inp[k] for k in PK]
    whole = gdn.kda_prefill(cfg, inp["qkv"], inp["zdec"], inp["b"], inp["gate"], inp["cu_seqlens"],
                            *P, initial_state=inp["initial_state"], return_final_state=True)
    cu = torch.tensor([0, T], dtype=torch.int32, device=cuda_device)
    part = gdn.kda_prefill(cfg, inp["qkv"][:T].contiguous(), inp["zdec"][:T].contiguous(),
                           inp["b"][:T].contiguous(), inp["gate"][:T].contiguous(), cu, *P,
                           initial_state=inp["initial_state"], return_final_state=True,
                           return_final_conv=True)
    S, Cc = part["final_state"].clone(), part["final_conv"].clone()
    y1 = gdn.kda_decode(cfg, inp["qkv"][T:].contiguous(), inp["zdec"][T:].contiguous(),
                        inp["b"][T:].contiguous(), inp["gate"][T:].contiguous(), S, Cc, *P)
    torch.cuda.synchronize()
    assert_output_close(torch.cat([part["y"], y1]), whole["y"], "continued y", rel=1e-3, mx=1e-2,
                        roundings=2)
    assert_state_close(S, whole["final_state"], "continued state", rel=1e-5)
