"""The workloads' layer shapes against the values the pages print (tests/golden/)."""
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
