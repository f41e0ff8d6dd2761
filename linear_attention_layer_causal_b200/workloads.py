"""Seeded synthetic workloads for the Gated DeltaNet token mixer.

This module only draws random inputs; it holds none of the layer's
arithmetic.  Both the CUDA library's callers and the CPU checker take their
inputs from here, so that both sides see identical bytes.

Shapes are the layer shapes the pages give: the Qwen3.8 Gated DeltaNet layer
(16 q/k heads, 128 value heads, head dim 128, conv kernel 4; "Qwen3.8 2.4T
A95B", raw config fields linear_num_key_heads, linear_num_value_heads,
linear_key_head_dim, linear_value_head_dim, linear_conv_kernel_dim), the
Qwen3.6-35B-A3B linear layer (16 key heads, 32 value heads; same page,
field-level comparison table) and the Qwen3.5-397B-A17B Gated DeltaNet layer
(16 q/k heads, 64 value heads, 4 per q/k head; "Qwen3.5-397B-A17B vs
Inkling", component table, Gated DeltaNet row).  No public dataset is
involved.

Distributions (all draws from one seeded generator, in the order listed):
  sequence lengths (varlen only) ~ integer U[lo, hi]
  qkv (pre-conv), a, b, z       ~ N(0, 1), cast to the activation dtype
  conv_w                        ~ N(0, 0.5^2)          (std 0.5)
  A_log                         = log U(1, 16)
  dt_bias                       ~ N(0, 0.5^2)
  norm_w                        = 1 + 0.1 N(0, 1)
  initial states                ~ N(0, 0.02^2) (where the workload has them)
  conv cache (decode)           ~ N(0, 1), activation dtype

Long-memory gates (gates="long_memory:<dt_bias>[:<b_mean>]"): A_log = 0 and
dt_bias = the given constant instead of the draws above, and b ~ N(b_mean,
0.5^2) (b_mean = 2 unless given), so that g = -softplus(a + dt_bias) is small
(about -0.018 per token at dt_bias = -4, -3e-4 at -8) and beta = sigmoid(b) is
about 0.88 (0.12 at b_mean = -2): the state keeps its past for hundreds to
thousands of tokens, where the default draws (exp(A_log) in [1, 16]) forget
within a few tokens.  A small beta also slows the delta rule's own erasure
along each new k, so the state carries across thousands of tokens.
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    num_qk_heads: int
    num_v_heads: int
    head_dim: int
    dtype: str = "bf16"                  # activation dtype: "bf16" or "f32"
    seqlens: tuple = ()                  # fixed sequence lengths (prefill)
    varlen: tuple | None = None          # (count, lo, hi): lengths ~ U[lo, hi] from the seed
    decode_batch: int = 0                # >0: one token per sequence against resident states
    state_std: float = 0.0               # initial-state std (0 = zero states)
    state_every: int = 1                 # sequences n with n % state_every == 0 get a state
    seed: int = 0
    conv_kernel: int = 4
    gates: str = "default"               # or "long_memory:<dt_bias>[:<b_mean>]" (module docstring)
    notes: str = field(default="", compare=False)

    @property
    def conv_dim(self) -> int:
        return (2 * self.num_qk_heads + self.num_v_heads) * self.head_dim

    @property
    def torch_dtype(self):
        return torch.bfloat16 if self.dtype == "bf16" else torch.float32


# The five workloads: a tiny bring-up layer, the Qwen3.8 layer in prefill
# (short and long), Qwen3.8 decode, and varlen prefill at the Qwen3.6-35B-A3B
# linear-layer shape.
TINY = Workload("tiny", 2, 4, 32, dtype="f32", seqlens=(128,), seed=1000,
                notes="B=1 T=128, 2 q/k heads, 4 value heads, d=32, fp32")
QWEN38_PREFILL = Workload("qwen38_prefill", 16, 128, 128, seqlens=(4096,), seed=1001,
                          notes="Qwen3.8 layer prefill, B=1 T=4096")
QWEN38_LONG = Workload("qwen38_long_prefill", 16, 128, 128, seqlens=(16384,) * 4,
                       state_std=0.02, seed=1002,
                       notes="Qwen3.8 layer prefill, B=4 T=16384, initial states")
QWEN38_DECODE = Workload("qwen38_decode", 16, 128, 128, decode_batch=256, state_std=0.02,
                         seed=1003, notes="Qwen3.8 layer decode, 256 sequences x 1 token")
QWEN36_VARLEN = Workload("qwen36_varlen", 16, 32, 128, varlen=(64, 256, 8192), state_std=0.02,
                         state_every=2, seed=1004,
                         notes="Qwen3.6-35B-A3B linear-layer shape, 64 packed sequences")

# Beyond the five: the Qwen3.5-397B-A17B layer shape (G = 4), and long-memory
# gates at the Qwen3.8 shape.
QWEN35_PREFILL = Workload("qwen35_prefill", 16, 64, 128, seqlens=(4096, 4096), state_std=0.02,
                          seed=1005, notes="Qwen3.5-397B-A17B layer prefill, B=2 T=4096")
QWEN35_DECODE = Workload("qwen35_decode", 16, 64, 128, decode_batch=256, state_std=0.02,
                         seed=1006, notes="Qwen3.5-397B-A17B layer decode, 256 sequences")
QWEN38_LONG_MEMORY = Workload("qwen38_long_memory", 16, 128, 128, seqlens=(16384,) * 3,
                              state_std=0.02, seed=1007, gates="long_memory:-4",
                              notes="Qwen3.8 layer, B=3 T=16384, slowly decaying state")
QWEN38_VERY_LONG_MEMORY = Workload("qwen38_very_long_memory", 16, 128, 128, seqlens=(16384,) * 3,
                                   state_std=0.02, seed=1008, gates="long_memory:-8",
                                   notes="Qwen3.8 layer, B=3 T=16384, nearly undecaying state")

# Long context: one sequence of 262,144 tokens, the Qwen3.8 context window
# ("Qwen3.8 2.4T A95B", key facts and raw config max_position_embeddings), at
# the Qwen3.8 layer shape and at the Qwen3.5-397B shape, whose 64 value heads
# leave more than half of the SMs to a split of the sequence.
QWEN38_262K = Workload("qwen38_262k_prefill", 16, 128, 128, seqlens=(262144,), seed=1010,
                       notes="Qwen3.8 layer, one 262,144-token sequence")
QWEN35_262K = Workload("qwen35_262k_prefill", 16, 64, 128, seqlens=(262144,), seed=1011,
                       notes="Qwen3.5-397B-A17B layer, one 262,144-token sequence")
# The sequence split under a state that carries across segments: nearly no
# decay and beta about 0.12; lengths with empty, one-token and ragged
# sequences beside ones of several segments.
SPLIT_MEMORY = Workload("qwen35_split_memory", 16, 64, 128, seqlens=(1100, 0, 593, 1, 2048),
                        state_std=0.02, seed=1012, gates="long_memory:-8:-2",
                        notes="Qwen3.5 layer, varlen, slowly forgetting state, for the split")

WORKLOADS = {w.name: w for w in (TINY, QWEN38_PREFILL, QWEN38_LONG, QWEN38_DECODE, QWEN36_VARLEN,
                                 QWEN35_PREFILL, QWEN35_DECODE, QWEN38_LONG_MEMORY,
                                 QWEN38_VERY_LONG_MEMORY, QWEN38_262K, QWEN35_262K,
                                 SPLIT_MEMORY)}  # (the KDA workload is added below)


def _gen(device, seed):
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    return g


def _normal(shape, std, g, device, dtype=torch.float32):
    x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    if std != 1.0:
        x.mul_(std)
    return x.to(dtype)


def _params(wl: Workload, g, device):
    H = wl.num_v_heads
    conv_w = _normal((wl.conv_dim, wl.conv_kernel), 0.5, g, device)
    A_log = torch.log(torch.rand(H, generator=g, device=device) * 15.0 + 1.0)
    dt_bias = _normal((H,), 0.5, g, device)
    norm_w = 1.0 + _normal((wl.head_dim,), 0.1, g, device)
    if wl.gates.startswith("long_memory"):
        A_log.zero_()
        dt_bias.fill_(float(wl.gates.split(":")[1]))
    return {"conv_w": conv_w.contiguous(), "A_log": A_log.contiguous(),
            "dt_bias": dt_bias.contiguous(), "norm_w": norm_w.contiguous()}


def seqlens_of(wl: Workload, g=None, device="cpu") -> list[int]:
    if wl.varlen is None:
        return list(wl.seqlens)
    count, lo, hi = wl.varlen
    g = g or _gen(device, wl.seed)
    return torch.randint(lo, hi + 1, (count,), generator=g, device=device).tolist()


def make_prefill(wl: Workload, device="cpu", seqlens=None, seed=None):
    """Inputs of one packed varlen prefill call.

    Returns a dict: qkv [N, conv_dim], a, b [N, H_v], z [N, H_v, d] (activation
    dtype), cu_seqlens [B+1] int32, conv_w [conv_dim, K], A_log, dt_bias [H_v],
    norm_w [d] (float32), initial_state [B, H_v, d, d] float32 or None, and
    seqlens (python list).  `seqlens` overrides the workload's lengths.
    """
    g = _gen(device, wl.seed if seed is None else seed)
    lens = seqlens_of(wl, g, device) if seqlens is None else list(seqlens)
    N = int(sum(lens))
    H, d, dt = wl.num_v_heads, wl.head_dim, wl.torch_dtype
    out = {"seqlens": lens}
    out["cu_seqlens"] = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()),
                                     dtype=torch.int32, device=device)
    out["qkv"] = _normal((N, wl.conv_dim), 1.0, g, device, dt)
    out["a"] = _normal((N, H), 1.0, g, device, dt)
    out["b"] = _normal((N, H), 1.0, g, device, dt)
    if wl.gates.startswith("long_memory"):
        parts = wl.gates.split(":")
        b_mean = float(parts[2]) if len(parts) > 2 else 2.0
        out["b"] = (out["b"].float() * 0.5 + b_mean).to(dt)
    out["z"] = _normal((N, H, d), 1.0, g, device, dt)
    out.update(_params(wl, g, device))
    if wl.state_std > 0:
        S = _normal((len(lens), H, d, d), wl.state_std, g, device)
        for n in range(len(lens)):
            if n % wl.state_every != 0:
                S[n].zero_()
        out["initial_state"] = S
    else:
        out["initial_state"] = None
    return out


def make_decode(wl: Workload, device="cpu", batch=None, seed=None, tokens=None):
    """Inputs of one decode call: one new token for each of B sequences.

    Returns qkv [B, conv_dim], a, b [B, H_v], z [B, H_v, d], conv_cache
    [B, K-1, conv_dim] (activation dtype), state [B, H_v, d, d] float32 and the
    float32 parameters.  With `tokens` = k, every sequence gets k new tokens
    instead: qkv [B, k, conv_dim], a, b [B, k, H_v], z [B, k, H_v, d].
    """
    g = _gen(device, wl.seed if seed is None else seed)
    B = batch or wl.decode_batch
    H, d, dt = wl.num_v_heads, wl.head_dim, wl.torch_dtype
    lead = (B,) if tokens is None else (B, tokens)
    out = {}
    out["qkv"] = _normal(lead + (wl.conv_dim,), 1.0, g, device, dt)
    out["a"] = _normal(lead + (H,), 1.0, g, device, dt)
    out["b"] = _normal(lead + (H,), 1.0, g, device, dt)
    out["z"] = _normal(lead + (H, d), 1.0, g, device, dt)
    out.update(_params(wl, g, device))
    out["state"] = _normal((B, H, d, d), wl.state_std if wl.state_std > 0 else 0.02, g, device)
    out["conv_cache"] = _normal((B, wl.conv_kernel - 1, wl.conv_dim), 1.0, g, device, dt)
    return out


# Kimi Delta Attention (per-channel decay) at the Kimi K3 layer shape: 96 heads
# of dimension 128, one q, k and v head each ("Inkling vs Kimi K3", component
# table, linear-attention row).  Draws, in order: lengths, qkv, the decay
# inputs zdec ~ N(0, 1), b ~ N(0, 1), the gate inputs ~ N(0, 1), conv_w ~
# N(0, 0.5^2), A_log = log U(1, 16), norm_w = 1 + 0.1 N(0, 1), states.
KIMI_K3_KDA = Workload("kimi_k3_kda", 96, 96, 128, seqlens=(1024, 517), state_std=0.02, seed=1009,
                       notes="Kimi K3 KDA layer prefill, B=2 (1024 + 517 tokens)")


def make_kda_prefill(wl: Workload, device="cpu", seqlens=None, seed=None):
    """Inputs of one KDA prefill call: qkv [N, 3 H d], zdec [N, H, d], b [N, H],
    gate [N, H, d], cu_seqlens, conv_w [3 H d, K], A_log [H], norm_w [d], and
    initial_state [B, H, d, d] or None."""
    g = _gen(device, wl.seed if seed is None else seed)
    lens = seqlens_of(wl, g, device) if seqlens is None else list(seqlens)
    N = int(sum(lens))
    H, d, dt = wl.num_v_heads, wl.head_dim, wl.torch_dtype
    out = {"seqlens": lens}
    out["cu_seqlens"] = torch.tensor([0] + list(torch.tensor(lens).cumsum(0).tolist()),
                                     dtype=torch.int32, device=device)
    out["qkv"] = _normal((N, wl.conv_dim), 1.0, g, device, dt)
    out["zdec"] = _normal((N, H, d), 1.0, g, device, dt)
    out["b"] = _normal((N, H), 1.0, g, device, dt)
    out["gate"] = _normal((N, H, d), 1.0, g, device, dt)
    out["conv_w"] = _normal((wl.conv_dim, wl.conv_kernel), 0.5, g, device).contiguous()
    out["A_log"] = torch.log(torch.rand(H, generator=g, device=device) * 15.0 + 1.0).contiguous()
    out["norm_w"] = (1.0 + _normal((d,), 0.1, g, device)).contiguous()
    out["initial_state"] = _normal((len(lens), H, d, d), wl.state_std, g, device) \
        if wl.state_std > 0 else None
    return out


def make_kda_decode(wl: Workload, device="cpu", batch=8, seed=None):
    """Inputs of one KDA decode call: one token for each of `batch` sequences."""
    g = _gen(device, wl.seed if seed is None else seed)
    H, d, dt = wl.num_v_heads, wl.head_dim, wl.torch_dtype
    out = {"qkv": _normal((batch, wl.conv_dim), 1.0, g, device, dt),
           "zdec": _normal((batch, H, d), 1.0, g, device, dt),
           "b": _normal((batch, H), 1.0, g, device, dt),
           "gate": _normal((batch, H, d), 1.0, g, device, dt),
           "conv_w": _normal((wl.conv_dim, wl.conv_kernel), 0.5, g, device).contiguous(),
           "A_log": torch.log(torch.rand(H, generator=g, device=device) * 15.0 + 1.0).contiguous(),
           "norm_w": (1.0 + _normal((d,), 0.1, g, device)).contiguous()}
    out["state"] = _normal((batch, H, d, d), 0.02, g, device)
    out["conv_cache"] = _normal((batch, wl.conv_kernel - 1, wl.conv_dim), 1.0, g, device, dt)
    return out

WORKLOADS[KIMI_K3_KDA.name] = KIMI_K3_KDA
