"""GPU parity: the CUDA library (through its C ABI) against the FP64 oracle.

Each test draws one seeded workload, runs the library on the device and the
oracle on the host over the same bytes, and compares element by element:
  - the small workloads in full,
  - the full-size workloads on sampled (sequence, q/k group, value head)
    units that the oracle computes one by one, plus whole-tensor properties
    (finite outputs, exact conv windows).
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


def _gpu_prefill(cfg, inp, **kw):
    kw.setdefault("check_status", True)
    return gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"],
                       *[inp[k] for k in PARAMS], initial_state=inp.get("initial_state"), **kw)


# the two prefill algorithms for head_dim 128: tensor-core chunks and token-serial
ALGOS = pytest.mark.parametrize("algo", ["chunked", "serial"])


def _oracle_seq(wl, inp, n, group=None, heads=None, conv=None):
    cu = inp["cu_seqlens"].tolist()
    s, e = cu[n], cu[n + 1]
    S0 = inp.get("initial_state")
    return oracle.layer(_shape(wl), inp["qkv"][s:e], inp["a"][s:e], inp["b"][s:e],
                        inp["z"][s:e], *[inp[k] for k in PARAMS],
                        state=None if S0 is None else S0[n],
                        conv_window=None if conv is None else conv[n], group=group, heads=heads)


def test_tiny_layer_full(cuda_device):
    """2 q/k heads, 4 value heads, d = 32, fp32 activations, T = 128: every output."""
    wl = W.TINY
    cfg = gdn.Config.of(wl)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_final_conv=True,
                       return_o_raw=True)
    torch.cuda.synchronize()
    ref = _oracle_seq(wl, inp, 0)
    assert_output_close(out["y"], ref["y"])
    assert_output_close(out["o_raw"], ref["o"], "o_raw")
    assert_state_close(out["final_state"][0], ref["state"])
    np.testing.assert_array_equal(to64(out["final_conv"][0]), ref["conv_window"])
    # fp32 operands throughout: far inside the bf16 tolerance
    assert_output_close(out["y"], ref["y"], rel=1e-4, mx=1e-3)
    assert_state_close(out["final_state"][0], ref["state"], rel=1e-4)


@ALGOS
def test_qwen38_prefill_all_heads(cuda_device, algo):
    """Qwen3.8 layer, B = 1, T = 4096, bf16: every value head against the oracle."""
    wl = W.QWEN38_PREFILL
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_final_conv=True,
                       return_o_raw=True)
    torch.cuda.synchronize()
    ref = _oracle_seq(wl, inp, 0)
    assert_output_close(out["y"], ref["y"])
    assert_output_close(out["o_raw"], ref["o"], "o_raw")
    assert_state_close(out["final_state"][0], ref["state"])
    np.testing.assert_array_equal(to64(out["final_conv"][0]), ref["conv_window"])


@ALGOS
def test_qwen38_long_prefill_sampled(cuda_device, algo):
    """Qwen3.8 layer, B = 4 x T = 16384 with N(0, 0.02) initial states: sampled heads."""
    wl = W.QWEN38_LONG
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_final_conv=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out["y"].float()).all()
    cu = inp["cu_seqlens"].tolist()
    G = wl.num_v_heads // wl.num_qk_heads
    # one whole q/k group (all G value heads) of each of three sequences
    for n, group in [(0, 0), (1, 9), (3, 15)]:
        heads = list(range(group * G, (group + 1) * G))
        ref = _oracle_seq(wl, inp, n, group)
        s, e = cu[n], cu[n + 1]
        r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n} group {group}")
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"qwen38_long[{algo}] seq {n} group {group}", r, m, rs)
    for n in range(len(cu) - 1):
        e = cu[n + 1]
        assert torch.equal(out["final_conv"][n], inp["qkv"][e - 3:e])


def test_qwen38_decode_sampled(cuda_device):
    """256 sequences x 1 token against resident N(0, 0.02) states: sampled sequences."""
    wl = W.QWEN38_DECODE
    cfg = gdn.Config.of(wl)
    inp = W.make_decode(wl, cuda_device)
    seqs = list(range(0, 256, 8)) + [1, 100, 255]
    S_before = inp["state"][seqs].cpu()
    C_before = inp["conv_cache"][seqs].cpu()
    y = gdn.decode(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["state"],
                   inp["conv_cache"], *[inp[k] for k in PARAMS])
    torch.cuda.synchronize()
    assert torch.isfinite(y.float()).all()
    sub = {k: (inp[k][seqs].cpu() if k in ("qkv", "a", "b", "z") else inp[k].cpu()) for k in
           ("qkv", "a", "b", "z") + PARAMS}
    ref = oracle.decode(_shape(wl), sub["qkv"], sub["a"], sub["b"], sub["z"],
                        *[sub[k] for k in PARAMS], state=S_before, conv_cache=C_before)
    r, m = assert_output_close(y[seqs], ref["y"])
    rs = assert_state_close(inp["state"][seqs], ref["state"])
    report(f"qwen38_decode ({len(seqs)} of 256 sequences)", r, m, rs)
    np.testing.assert_array_equal(to64(inp["conv_cache"][seqs]), ref["conv_window"])


@ALGOS
def test_qwen36_varlen_sampled(cuda_device, algo):
    """64 packed sequences with lengths U[256, 8192], 16 q/k / 32 value heads: sampled units."""
    wl = W.QWEN36_VARLEN
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    lens = inp["seqlens"]
    out = _gpu_prefill(cfg, inp, return_final_state=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out["y"].float()).all()
    cu = inp["cu_seqlens"].tolist()
    order = np.argsort(lens)
    # shortest, longest, with and without an initial state; each pick checks one
    # whole q/k group (both of its value heads)
    picks = [(int(order[0]), 0), (int(order[-1]), 15), (2, 7), (5, 3), (int(order[32]), 11)]
    for n, group in picks:
        ref = _oracle_seq(wl, inp, n, group)
        s, e = cu[n], cu[n + 1]
        heads = [2 * group, 2 * group + 1]
        r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n} (len {lens[n]})")
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"qwen36_varlen[{algo}] seq {n} len {lens[n]} group {group}", r, m, rs)


EDGE = W.Workload("edge", 2, 4, 128, seqlens=(0, 1, 2, 3, 5, 33, 64, 0, 100, 31), state_std=0.02,
                  seed=77)


@ALGOS
@pytest.mark.parametrize("with_conv", [False, True])
def test_edge_lengths_full(cuda_device, with_conv, algo):
    """Empty, shorter-than-window and ragged sequences, with and without incoming conv windows."""
    wl = EDGE
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    B = len(wl.seqlens)
    conv = None
    if with_conv:
        g = torch.Generator(device=cuda_device).manual_seed(5)
        conv = torch.randn((B, 3, wl.conv_dim), generator=g, device=cuda_device).to(torch.bfloat16)
    out = _gpu_prefill(cfg, inp, initial_conv=conv, return_final_state=True,
                       return_final_conv=True, return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    for n in range(B):
        ref = _oracle_seq(wl, inp, n, conv=conv)
        s, e = cu[n], cu[n + 1]
        if e > s:
            assert_output_close(out["y"][s:e], ref["y"], f"y seq {n}")
            assert_output_close(out["o_raw"][s:e], ref["o"], f"o seq {n}")
        assert_state_close(out["final_state"][n], ref["state"], f"state seq {n}")
        np.testing.assert_array_equal(to64(out["final_conv"][n]), ref["conv_window"])
    # empty sequences pass their state through exactly
    for n in (0, 7):
        assert torch.equal(out["final_state"][n], inp["initial_state"][n])


@ALGOS
@pytest.mark.parametrize("shape", [(1, 3), (3, 9)], ids=["1x3", "3x9"])
def test_odd_value_head_count(cuda_device, shape, algo):
    """An odd number of value heads (G = 3): the inverse kernel's CTAs take two
    value heads each, so the last one has an idle half.  Every head of two
    ragged sequences against the oracle."""
    Hk, Hv = shape
    wl = W.Workload(f"odd_heads_{Hk}x{Hv}", Hk, Hv, 128, seqlens=(70, 129), state_std=0.02, seed=23)
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    for n in range(len(wl.seqlens)):
        ref = _oracle_seq(wl, inp, n)
        s, e = cu[n], cu[n + 1]
        r, m = assert_output_close(out["y"][s:e], ref["y"], f"y seq {n}")
        assert_output_close(out["o_raw"][s:e], ref["o"], f"o seq {n}")
        rs = assert_state_close(out["final_state"][n], ref["state"], f"state seq {n}")
        report(f"{wl.name} {algo} seq {n}", r, m, rs)


EDGE_F32 = W.Workload("edge_f32", 2, 4, 128, dtype="f32", seqlens=(0, 5, 64, 100, 31),
                      state_std=0.02, seed=78)


@ALGOS
def test_float32_activations_head_dim_128(cuda_device, algo):
    """fp32 activations at head dim 128 (the float instantiation of every kernel of both
    paths), with empty and ragged sequences."""
    wl = EDGE_F32
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    assert inp["qkv"].dtype == torch.float32
    B = len(wl.seqlens)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    for n in range(B):
        ref = _oracle_seq(wl, inp, n)
        s, e = cu[n], cu[n + 1]
        if e > s:
            assert_output_close(out["y"][s:e], ref["y"], f"y seq {n}")
            assert_output_close(out["o_raw"][s:e], ref["o"], f"o seq {n}")
        assert_state_close(out["final_state"][n], ref["state"], f"state seq {n}")


@ALGOS
def test_in_place_state_and_conv(cuda_device, algo):
    """final_state = initial_state and final_conv = initial_conv give the out-of-place result."""
    wl = EDGE
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    B = len(wl.seqlens)
    g = torch.Generator(device=cuda_device).manual_seed(6)
    conv = torch.randn((B, 3, wl.conv_dim), generator=g, device=cuda_device).to(torch.bfloat16)
    ref = _gpu_prefill(cfg, inp, initial_conv=conv, return_final_state=True,
                       return_final_conv=True)
    S = inp["initial_state"].clone()
    C = conv.clone()
    inp2 = dict(inp, initial_state=S)
    out = _gpu_prefill(cfg, inp2, initial_conv=C, final_state=S, final_conv=C)
    torch.cuda.synchronize()
    assert torch.equal(out["y"], ref["y"])
    assert torch.equal(S, ref["final_state"])
    assert torch.equal(C, ref["final_conv"])


@ALGOS
def test_split_prefill_and_decode_continue_the_sequence(cuda_device, algo):
    """prefill [0, T1) + prefill [T1, T) with carried state and conv window, then decode one
    token, equals prefill [0, T + 1) -- all on the device."""
    wl = W.Workload("cont", 4, 16, 128, seqlens=(301,), state_std=0.02, seed=91)
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    T1, T = 130, 300
    P = [inp[k] for k in PARAMS]
    whole = gdn.prefill(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["cu_seqlens"], *P,
                        initial_state=inp["initial_state"], return_final_state=True)

    def part(s, e, S0, C0):
        cu = torch.tensor([0, e - s], dtype=torch.int32, device=cuda_device)
        return gdn.prefill(cfg, inp["qkv"][s:e].contiguous(), inp["a"][s:e].contiguous(),
                           inp["b"][s:e].contiguous(), inp["z"][s:e].contiguous(), cu, *P,
                           initial_state=S0, initial_conv=C0, return_final_state=True,
                           return_final_conv=True)
    p1 = part(0, T1, inp["initial_state"], None)
    p2 = part(T1, T, p1["final_state"], p1["final_conv"])
    state = p2["final_state"].clone()
    cache = p2["final_conv"].clone()
    y1 = gdn.decode(cfg, inp["qkv"][T:T + 1].contiguous(), inp["a"][T:T + 1].contiguous(),
                    inp["b"][T:T + 1].contiguous(), inp["z"][T:T + 1].contiguous(), state,
                    cache, *P)
    torch.cuda.synchronize()
    ys = torch.cat([p1["y"], p2["y"], y1])
    # the two runs split the sequence at different chunk boundaries, so with
    # tf32 products they agree to rounding level only
    tight = algo == "serial"
    assert_output_close(ys, whole["y"], "continued y", rel=2e-3 if tight else 5e-3,
                        mx=1e-2 if tight else 2e-2)
    assert_state_close(state, whole["final_state"], "continued state", rel=1e-4 if tight else 2e-3)
    assert torch.equal(cache[0], inp["qkv"][T - 2:T + 1])


@ALGOS
@pytest.mark.parametrize("wl", [W.QWEN38_LONG_MEMORY, W.QWEN38_VERY_LONG_MEMORY],
                         ids=lambda w: w.name)
def test_long_memory_full_groups(cuda_device, wl, algo):
    """Slowly decaying states (A_log = 0, dt_bias = -4 or -8, beta ~ 0.88) over
    B = 3 x T = 16384: the state carries its past across hundreds of chunks, so
    any bias in the chunked path's operand rounding would accumulate instead of
    being forgotten within a chunk.  One whole q/k group of each sequence,
    element by element against the oracle, with the stated bounds."""
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_o_raw=True)
    torch.cuda.synchronize()
    cu = inp["cu_seqlens"].tolist()
    G = wl.num_v_heads // wl.num_qk_heads
    for n, group in [(0, 3), (1, 8), (2, 14)]:
        heads = list(range(group * G, (group + 1) * G))
        ref = _oracle_seq(wl, inp, n, group)
        s, e = cu[n], cu[n + 1]
        r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n} group {group}")
        ro, mo = assert_output_close(out["o_raw"][s:e, heads], ref["o"], f"o seq {n}")
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"{wl.name}[{algo}] seq {n} group {group}", r, m, rs)
        report(f"{wl.name}[{algo}] seq {n} group {group} o_raw", ro, mo)


@ALGOS
def test_all_sequences_empty(cuda_device, algo):
    """A batch of sequences with no tokens at all: nothing is computed, every state
    and conv window passes through unchanged, and no workspace is needed."""
    wl = W.Workload("empty", 2, 4, 128, seqlens=(0, 0, 0), state_std=0.02, seed=5)
    cfg = gdn.Config.of(wl, algo)
    assert gdn.prefill_workspace_size(cfg, 3, 0) == 0
    inp = W.make_prefill(wl, cuda_device)
    g = torch.Generator(device=cuda_device).manual_seed(9)
    conv = torch.randn((3, 3, wl.conv_dim), generator=g, device=cuda_device).to(torch.bfloat16)
    out = _gpu_prefill(cfg, inp, initial_conv=conv, return_final_state=True,
                       return_final_conv=True, check_status=False)
    torch.cuda.synchronize()
    assert out["y"].numel() == 0
    assert torch.equal(out["final_state"], inp["initial_state"])
    assert torch.equal(out["final_conv"], conv)


def test_bounded_wait_timeout_aborts_cleanly(cuda_device):
    """A wait between the chunk kernel's warps that runs out (here: forced by a
    limit of 100 SM cycles, far below any real hand-over) makes the call abort
    without a fault or a hang: the status query reports GDN_ERR_TIMEOUT, and the
    next call on the same workspace and context is clean and correct."""
    wl = W.Workload("timeout", 1, 2, 128, seqlens=(300, 77), state_std=0.02, seed=17)
    cfg = gdn.Config.of(wl, "chunked")
    inp = W.make_prefill(wl, cuda_device)
    B, N = 2, 377
    ws = torch.empty(gdn.prefill_workspace_size(cfg, B, N), dtype=torch.uint8, device=cuda_device)
    ref = _gpu_prefill(cfg, inp, return_final_state=True, workspace=ws)
    assert gdn.prefill_status(ws) == (gdn.GDN_OK, 0)
    gdn.wait_limit_next_call(100)
    _gpu_prefill(cfg, inp, return_final_state=True, workspace=ws, check_status=False)
    st, detail = gdn.prefill_status(ws)
    assert st == gdn.GDN_ERR_TIMEOUT
    assert detail == 0 or (detail & 0x80000000), f"detail {detail:#x}"
    again = _gpu_prefill(cfg, inp, return_final_state=True, workspace=ws)
    torch.cuda.synchronize()
    assert gdn.prefill_status(ws) == (gdn.GDN_OK, 0)
    assert torch.equal(again["y"], ref["y"])
    assert torch.equal(again["final_state"], ref["final_state"])


@ALGOS
def test_qwen35_prefill_sampled_groups(cuda_device, algo):
    """The Qwen3.5-397B-A17B layer shape (16 q/k heads, 64 value heads, G = 4),
    B = 2 x T = 4096 with initial states: whole q/k groups against the oracle."""
    wl = W.QWEN35_PREFILL
    cfg = gdn.Config.of(wl, algo)
    inp = W.make_prefill(wl, cuda_device)
    out = _gpu_prefill(cfg, inp, return_final_state=True, return_final_conv=True)
    torch.cuda.synchronize()
    assert torch.isfinite(out["y"].float()).all()
    cu = inp["cu_seqlens"].tolist()
    for n, group in [(0, 0), (0, 10), (1, 5), (1, 15)]:
        heads = list(range(4 * group, 4 * group + 4))
        ref = _oracle_seq(wl, inp, n, group)
        s, e = cu[n], cu[n + 1]
        r, m = assert_output_close(out["y"][s:e, heads], ref["y"], f"y seq {n} group {group}")
        rs = assert_state_close(out["final_state"][n, heads], ref["state"], f"state seq {n}")
        report(f"qwen35_prefill[{algo}] seq {n} group {group}", r, m, rs)
    for n in range(2):
        assert torch.equal(out["final_conv"][n], inp["qkv"][cu[n + 1] - 3:cu[n + 1]])


def test_qwen35_decode_sampled(cuda_device):
    """Decode at the Qwen3.5-397B-A17B shape: 256 sequences, sampled ones against the oracle."""
    wl = W.QWEN35_DECODE
    cfg = gdn.Config.of(wl)
    inp = W.make_decode(wl, cuda_device)
    seqs = [0, 31, 128, 255]
    S_before = inp["state"][seqs].cpu()
    C_before = inp["conv_cache"][seqs].cpu()
    y = gdn.decode(cfg, inp["qkv"], inp["a"], inp["b"], inp["z"], inp["state"],
                   inp["conv_cache"], *[inp[k] for k in PARAMS])
    torch.cuda.synchronize()
    sub = {k: inp[k][seqs].cpu() for k in ("qkv", "a", "b", "z")}
    ref = oracle.decode(_shape(wl), sub["qkv"], sub["a"], sub["b"], sub["z"],
                        *[inp[k].cpu() for k in PARAMS], state=S_before, conv_cache=C_before)
    r, m = assert_output_close(y[seqs], ref["y"])
    rs = assert_state_close(inp["state"][seqs], ref["state"])
    report("qwen35_decode", r, m, rs)
    np.testing.assert_array_equal(to64(inp["conv_cache"][seqs]), ref["conv_window"])
