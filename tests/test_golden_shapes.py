"""The workloads' layer shapes and lengths against the values the pages print (tests/golden/)."""
import os

from linear_attention_layer_causal_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split()
            out[k] = v
    return out


def test_qwen38_shape():
    g = _read("qwen38_gdn_layer_shape.txt")
    for wl in (W.QWEN38_PREFILL, W.QWEN38_LONG, W.QWEN38_DECODE):
        assert wl.num_qk_heads == int(g["linear_num_key_heads"])
        assert wl.num_v_heads == int(g["linear_num_value_heads"])
        assert wl.head_dim == int(g["linear_key_head_dim"]) == int(g["linear_value_head_dim"])
        assert wl.conv_kernel == int(g["linear_conv_kernel_dim"])
        assert wl.num_v_heads // wl.num_qk_heads == int(g["value_heads_per_qk_head"])
        assert wl.num_v_heads * wl.head_dim ** 2 == int(g["state_floats_per_sequence"])
    assert float(g["rms_norm_eps"]) == 1e-6


def test_qwen36_shape():
    g = _read("qwen36_linear_layer_shape.txt")
    wl = W.QWEN36_VARLEN
    assert wl.num_qk_heads == int(g["linear_num_key_heads"])
    assert wl.num_v_heads == int(g["linear_num_value_heads"])
    assert wl.head_dim == int(g["linear_key_head_dim"])
    assert wl.conv_kernel == int(g["linear_conv_kernel_dim"])


def test_qwen35_shape():
    g = _read("qwen35_gdn_layer_shape.txt")
    for wl in (W.QWEN35_PREFILL, W.QWEN35_DECODE, W.QWEN35_262K, W.SPLIT_MEMORY):
        assert wl.num_qk_heads == int(g["linear_num_key_heads"])
        assert wl.num_v_heads == int(g["linear_num_value_heads"])
        assert wl.head_dim == int(g["head_dim"])
        assert wl.conv_kernel == int(g["conv_kernel"])
        assert wl.num_v_heads // wl.num_qk_heads == int(g["value_heads_per_qk_head"])
        assert wl.num_v_heads * wl.head_dim ** 2 == int(g["state_floats_per_sequence"])


def test_kimi_k3_kda_shape_and_decay_bound():
    g = _read("kimi_k3_kda_layer_shape.txt")
    wl = W.KIMI_K3_KDA
    assert wl.num_qk_heads == wl.num_v_heads == int(g["num_heads"])  # one q/k per head
    assert wl.head_dim == int(g["head_dim"])
    assert wl.conv_kernel == int(g["conv_kernel"])
    assert wl.num_v_heads * wl.head_dim ** 2 == int(g["state_floats_per_sequence"])
    # the oracle's per-channel log-decay tends to the printed bound at large
    # positive e^A z, to 0 at large negative, and stays inside (-bound, 0)
    import numpy as np

    import oracle
    bound = float(g["log_decay_bound"])
    z = np.array([[[60.0, -60.0, 0.0, 1.5]]])
    dec, _ = oracle.kda_gates(z, np.zeros((1, 1)), np.array([0.0]))
    assert abs(dec[0, 0, 0] + bound) < 1e-12 and abs(dec[0, 0, 1]) < 1e-12
    assert np.all(dec[0, 0, 2:] > -bound) and np.all(dec[0, 0, 2:] < 0)
    assert dec[0, 0, 2] == -bound / 2  # sigmoid(0) = 1/2


def test_long_context_workloads_span_the_context_window():
    g = _read("qwen38_context.txt")
    n = int(g["max_position_embeddings"])
    assert W.QWEN38_262K.seqlens == (n,)
    assert W.QWEN35_262K.seqlens == (n,)
