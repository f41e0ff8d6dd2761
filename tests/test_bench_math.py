"""The bench's roofline denominators, checked on the CPU against the tensors
they count: the algorithmic bytes of prefill, decode and KDA decode equal the
bytes of the inputs a call must read and the outputs it must write (from the
seeded generators' own tensors), and the chunked-form FLOPs per token add up
the products of one chunk."""
import importlib
import os
import sys

import pytest
import torch

from linear_attention_layer_causal_b200 import workloads as W

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
bench = importlib.import_module("bench")


def _nbytes(*ts):
    return sum(t.numel() * t.element_size() for t in ts)


@pytest.mark.parametrize("shape", [(2, 4, 32), (4, 16, 128)])
def test_prefill_bytes_are_the_call_inputs_and_outputs(shape):
    Hk, Hv, d = shape
    wl = W.Workload("b", Hk, Hv, d, seqlens=(5, 0, 11), seed=1)
    inp = W.make_prefill(wl)
    N, B = 16, 3
    y = torch.empty((N, Hv, d), dtype=wl.torch_dtype)
    state = torch.empty((B, Hv, d, d), dtype=torch.float32)
    reads = _nbytes(inp["qkv"], inp["z"], inp["a"], inp["b"])
    assert bench.prefill_bytes(Hk, Hv, d, N, B) == reads + _nbytes(y, state)
    assert bench.prefill_bytes(Hk, Hv, d, N, B, read_state=True) == reads + _nbytes(y) + 2 * _nbytes(state)


def test_decode_bytes_are_the_call_inputs_and_outputs():
    wl = W.Workload("d", 4, 16, 128, decode_batch=3, state_std=0.02, seed=2)
    inp = W.make_decode(wl)
    y = torch.empty_like(inp["z"])
    # state and conv cache are read and written back; the token rows are read, y written
    want = 2 * _nbytes(inp["state"], inp["conv_cache"]) + _nbytes(inp["qkv"], inp["z"], inp["a"], inp["b"], y)
    assert bench.decode_bytes(4, 16, 128, 3) == want


def test_kda_decode_bytes_are_the_call_inputs_and_outputs():
    wl = W.Workload("k", 6, 6, 128, seed=3)
    inp = W.make_kda_decode(wl, batch=2)
    y = torch.empty_like(inp["gate"])
    want = 2 * _nbytes(inp["state"], inp["conv_cache"]) + \
        _nbytes(inp["qkv"], inp["zdec"], inp["gate"], inp["b"], y)
    assert bench.kda_decode_bytes(6, 128, 2) == want


def test_chunked_flops_add_up_one_chunk():
    Hk, Hv, d, C = 16, 128, 128, 64

    def mm(m, n, k):
        return 2 * m * n * k

    per_v = (mm(C, d, C)            # U~ = T diag(beta) V
             + mm(C, d, C)          # W = T diag(beta gamma) K
             + mm(C, d, d)          # W S0^T
             + mm(C, d, d)          # Q S0^T
             + mm(d, d, C)          # the state update U^T K
             + mm(C, d, C)          # P U
             + C ** 3 / 3)          # T = (I + A)^-1 by substitution
    per_k = mm(C, C, d) * 2         # K K^T and Q K^T
    per_chunk = Hv * per_v + Hk * per_k
    assert bench.prefill_flops_per_token(Hk, Hv, d) * C == pytest.approx(per_chunk, rel=1e-12)
    # one 4,096-token call: 80.17 GFLOP
    assert bench.prefill_flops_per_token(Hk, Hv, d) * 4096 == pytest.approx(80.17e9, rel=1e-3)
