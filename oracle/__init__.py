"""FP64 CPU oracle of the Gated DeltaNet token mixer.

TEST INFRASTRUCTURE ONLY.  This package is the checker that the CUDA library
is compared against: only the tests, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg may import it.  It shares no code with the CUDA
path (``linear_attention_layer_causal_b200``) and imports nothing from it.

The arithmetic lives in ``gdn_oracle.c`` (plain C, FP64, one token at a
time); this module widens inputs to float64, calls the C stages in the order
the layer defines, and composes them into a whole prefill or decode pass:

    conv+SiLU over q|k|v  ->  L2-normalise q, k per q/k head  ->  gates
    ->  gated delta rule per value head (value head h reads q/k head h // G)
    ->  per-head RMSNorm times weight times SiLU(z)

(Gated DeltaNet row and output-gate row of the component table on
"Qwen3.8-2.4T-A95B vs Inkling"; head counts, kernel size, state dtype and
epsilon from the raw config fields on "Qwen3.8 2.4T A95B".)

The KDA variant (kda_layer, kda_prefill) swaps the gates, the recurrence and
the output gate for the per-key-channel decay g = -5 sigmoid(exp(A_log) z),
S_t = S_{t-1} Diag(exp(g_t)) (I - beta k k^T) + beta v k^T, and y = RMSNorm(o)
w sigmoid(gate) ("Inkling vs Kimi K3", component table, linear-attention and
output-gate rows); q, k and v go through the same conv, SiLU and L2 norm.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_SO = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64 = ctypes.c_int64


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdn_oracle.so beside it (gcc, -O2, pthreads)."""
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c99", "-D_POSIX_C_SOURCE=200809L", "-fPIC", "-shared",
             "-fno-fast-math", "-ffp-contract=off", "-o", tmp, _SRC, "-lm", "-lpthread"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(_SO)
        L.gdn_oracle_conv_silu.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _dp]
        L.gdn_oracle_conv_silu.restype = None
        L.gdn_oracle_l2norm_rows.argtypes = [_dp, _i64, _i64, ctypes.c_double, ctypes.c_double]
        L.gdn_oracle_l2norm_rows.restype = None
        L.gdn_oracle_gates.argtypes = [_dp, _dp, _dp, _dp, _i64, _i64, _dp, _dp]
        L.gdn_oracle_gates.restype = None
        L.gdn_oracle_delta_rule.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64,
                                            _i64, _dp, _dp, ctypes.c_int]
        L.gdn_oracle_delta_rule.restype = ctypes.c_int
        L.gdn_oracle_gated_rmsnorm.argtypes = [_dp, _dp, _dp, _i64, _i64, ctypes.c_double, _dp]
        L.gdn_oracle_gated_rmsnorm.restype = None
        L.gdn_oracle_kda_gates.argtypes = [_dp, _dp, _dp, _i64, _i64, _i64, _dp, _dp]
        L.gdn_oracle_kda_gates.restype = None
        L.gdn_oracle_kda_rule.argtypes = [_dp, _dp, _dp, _dp, _dp, _i64, _i64, _i64, _i64, _dp,
                                          _dp, ctypes.c_int]
        L.gdn_oracle_kda_rule.restype = None
        L.gdn_oracle_sigmoid_rmsnorm.argtypes = [_dp, _dp, _dp, _i64, _i64, ctypes.c_double, _dp]
        L.gdn_oracle_sigmoid_rmsnorm.restype = None
        _lib = L
    return _lib


def _f64(x) -> np.ndarray:
    """Exact widening of a numpy array or a (CPU or CUDA) torch tensor to C-contiguous float64."""
    if hasattr(x, "detach"):
        x = x.detach().to("cpu").double().numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _take(x, idx, axis: int = 1) -> np.ndarray:
    """x[..., idx, ...] along `axis`, sliced before widening so large inputs stay small."""
    if hasattr(x, "detach"):
        import torch
        ti = torch.as_tensor(np.asarray(idx, dtype=np.int64), device=x.device)
        return _f64(x.index_select(axis, ti))
    return _f64(np.take(np.asarray(x), np.asarray(idx, dtype=np.int64), axis=axis))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    assert a.dtype == np.float64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_dp)


def default_threads() -> int:
    return len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)


# ---------------------------------------------------------------- stages


def conv_silu(x, w, window=None) -> np.ndarray:
    """Depthwise causal conv (w[:, -1] on the current token, no bias) + SiLU.

    x: [T, C]; w: [C, K]; window: [K-1, C] previous rows, oldest first (None = zeros).
    """
    x, w = _f64(x), _f64(w)
    T, C = x.shape
    K = w.shape[1]
    win = None if window is None else _f64(window)
    if win is not None:
        assert win.shape == (K - 1, C)
    out = np.empty((T, C), np.float64)
    lib().gdn_oracle_conv_silu(_ptr(x), _ptr(win), _ptr(w), T, C, K, _ptr(out))
    return out


def l2norm(x, eps: float = 1e-6, scale: float = 1.0) -> np.ndarray:
    """Each length-d row (last axis) divided by sqrt(sum of squares + eps), times scale."""
    x = _f64(x).copy()
    d = x.shape[-1]
    lib().gdn_oracle_l2norm_rows(_ptr(x), x.size // d, d, eps, scale)
    return x


def gates(a, b, A_log, dt_bias):
    """g = -exp(A_log) * softplus(a + dt_bias), beta = sigmoid(b); a, b: [T, H]."""
    a, b, A_log, dt_bias = _f64(a), _f64(b), _f64(A_log), _f64(dt_bias)
    T, H = a.shape
    g = np.empty((T, H), np.float64)
    beta = np.empty((T, H), np.float64)
    lib().gdn_oracle_gates(_ptr(a), _ptr(b), _ptr(A_log), _ptr(dt_bias), T, H, _ptr(g), _ptr(beta))
    return g, beta


def delta_rule(q, k, v, g, beta, state=None, threads: int | None = None):
    """Gated delta rule over one sequence.

    q, k: [T, H_k, d_k]; v: [T, H_v, d_v]; g, beta: [T, H_v];
    state: [H_v, d_v, d_k] initial state (None = zeros).
    Returns (o [T, H_v, d_v], final state [H_v, d_v, d_k]).
    """
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    T, H_k, d_k = k.shape
    _, H_v, d_v = v.shape
    S = np.zeros((H_v, d_v, d_k)) if state is None else _f64(state).copy()
    o = np.empty((T, H_v, d_v), np.float64)
    rc = lib().gdn_oracle_delta_rule(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H_k, H_v,
                                     d_k, d_v, _ptr(S), _ptr(o), threads or default_threads())
    if rc != 0:
        raise ValueError("value heads must be a multiple of q/k heads")
    return o, S


def gated_rmsnorm(o, z, w, eps: float = 1e-6) -> np.ndarray:
    """y = o / sqrt(mean(o^2) + eps) * w * SiLU(z), over the last axis."""
    o, z, w = _f64(o), _f64(z), _f64(w)
    d = o.shape[-1]
    y = np.empty_like(o)
    lib().gdn_oracle_gated_rmsnorm(_ptr(o), _ptr(z), _ptr(w), o.size // d, d, eps, _ptr(y))
    return y


# ---------------------------------------------------------------- layer


@dataclass
class Shape:
    """Head layout of one layer: H_k q/k heads and H_v value heads, all of dim d."""
    num_qk_heads: int
    num_v_heads: int
    head_dim: int
    conv_kernel: int = 4
    rms_eps: float = 1e-6
    l2_eps: float = 1e-6
    q_scale: float = 1.0

    @property
    def conv_dim(self) -> int:
        return (2 * self.num_qk_heads + self.num_v_heads) * self.head_dim


def _group_columns(shape: Shape, group: int, heads):
    """Pre-conv channel indices of q/k head `group` and of the value heads `heads`."""
    d, Hk = shape.head_dim, shape.num_qk_heads
    qc = np.arange(group * d, (group + 1) * d)
    kc = Hk * d + qc
    vc = np.concatenate([2 * Hk * d + h * d + np.arange(d) for h in heads]) if len(heads) else \
        np.zeros(0, np.int64)
    return qc, kc, vc


def layer(shape: Shape, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w,
          state=None, conv_window=None, group: int | None = None, heads=None,
          threads: int | None = None):
    """One sequence through the whole mixer.

    qkv: [T, conv_dim] pre-conv rows; a, b: [T, H_v]; z: [T, H_v, d];
    conv_w: [conv_dim, K]; A_log, dt_bias: [H_v]; norm_w: [d];
    state: [H_v, d, d] (None = zeros); conv_window: [K-1, conv_dim] (None = zeros).

    With `group` set, only q/k head `group` and the value heads `heads` (a
    subset of that group's value heads; all of them if None) are computed,
    and every per-value-head output holds just those heads, in that order.
    Returns a dict with y, o (pre-norm), state (final) and conv_window (final:
    the last K-1 pre-conv rows of [conv_window; qkv]).
    """
    d, Hk, Hv, K = shape.head_dim, shape.num_qk_heads, shape.num_v_heads, shape.conv_kernel
    G = Hv // Hk
    qkv_t = qkv
    T = int(qkv.shape[0])
    if group is None:
        heads = list(range(Hv))
        cols = None
        n_qk = Hk
    else:
        heads = list(range(group * G, (group + 1) * G)) if heads is None else list(heads)
        assert all(h // G == group for h in heads)
        qc, kc, vc = _group_columns(shape, group, heads)
        cols = np.concatenate([qc, kc, vc])
        n_qk = 1
    hv = len(heads)
    # widen only the columns this call needs
    if cols is None:
        x = _f64(qkv_t)
        w = _f64(conv_w)
        win = None if conv_window is None else _f64(conv_window)
    else:
        x = _take(qkv_t, cols, 1)
        w = _take(conv_w, cols, 0)
        win = None if conv_window is None else _take(conv_window, cols, 1)
    xc = conv_silu(x, w, win)
    q = l2norm(xc[:, : n_qk * d].reshape(T, n_qk, d), shape.l2_eps, shape.q_scale)
    k = l2norm(xc[:, n_qk * d: 2 * n_qk * d].reshape(T, n_qk, d), shape.l2_eps, 1.0)
    v = xc[:, 2 * n_qk * d:].reshape(T, hv, d)
    a64, b64 = _take(a, heads, 1), _take(b, heads, 1)
    g, beta = gates(a64, b64, _take(A_log, heads, 0), _take(dt_bias, heads, 0))
    S0 = None if state is None else _take(state, heads, 0)
    o, S = delta_rule(q, k, v, g, beta, S0, threads)
    zz = _take(z, heads, 1)
    y = gated_rmsnorm(o, zz, norm_w, shape.rms_eps)
    # final conv window: last K-1 rows of [window; x] over this call's columns
    prev = np.zeros((K - 1, x.shape[1])) if win is None else win
    hist = np.concatenate([prev, x], axis=0)
    return {"y": y, "o": o, "state": S, "conv_window": hist[-(K - 1):].copy(),
            "g": g, "beta": beta, "q": q, "k": k, "v": v}


def prefill(shape: Shape, qkv, a, b, z, cu_seqlens, conv_w, A_log, dt_bias, norm_w,
            initial_state=None, initial_conv=None, threads: int | None = None):
    """Packed varlen prefill: sequence n is rows cu_seqlens[n]:cu_seqlens[n+1].

    initial_state: [B, H_v, d, d] or None; initial_conv: [B, K-1, conv_dim] or None.
    Returns y [N, H_v, d], o [N, H_v, d], state [B, H_v, d, d], conv [B, K-1, conv_dim].
    """
    cu = [int(c) for c in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    B = len(cu) - 1
    d, Hv, K = shape.head_dim, shape.num_v_heads, shape.conv_kernel
    N = cu[-1]
    y = np.empty((N, Hv, d))
    o = np.empty((N, Hv, d))
    S = np.empty((B, Hv, d, d))
    cw = np.empty((B, K - 1, shape.conv_dim))
    for n in range(B):
        s, e = cu[n], cu[n + 1]
        r = layer(shape, qkv[s:e], a[s:e], b[s:e], z[s:e], conv_w, A_log, dt_bias, norm_w,
                  None if initial_state is None else initial_state[n],
                  None if initial_conv is None else initial_conv[n], threads=threads)
        y[s:e], o[s:e], S[n], cw[n] = r["y"], r["o"], r["state"], r["conv_window"]
    return {"y": y, "o": o, "state": S, "conv_window": cw}


def decode(shape: Shape, qkv, a, b, z, conv_w, A_log, dt_bias, norm_w, state, conv_cache,
           seqs=None, threads: int | None = None):
    """One new token for each sequence against its resident state and conv cache.

    qkv: [B, conv_dim]; a, b: [B, H_v]; z: [B, H_v, d]; state: [B, H_v, d, d];
    conv_cache: [B, K-1, conv_dim].  Decoding is the one-token case of the
    layer: the token's conv window is the cache, and the new cache drops the
    oldest row and appends the token's pre-conv row.  `seqs` limits the work
    to those sequences (outputs stacked in that order).
    """
    B = qkv.shape[0]
    seqs = list(range(B)) if seqs is None else list(seqs)
    outs = []
    for n in seqs:
        outs.append(layer(shape, qkv[n:n + 1], a[n:n + 1], b[n:n + 1], z[n:n + 1], conv_w, A_log,
                          dt_bias, norm_w, state[n], conv_cache[n], threads=threads))
    return {"y": np.concatenate([r["y"] for r in outs]),
            "o": np.concatenate([r["o"] for r in outs]),
            "state": np.stack([r["state"] for r in outs]),
            "conv_window": np.stack([r["conv_window"] for r in outs])}


# ---------------------------------------------------------------- KDA


def kda_gates(z, b, A_log):
    """g = -5 sigmoid(exp(A_log) z) per key channel, beta = sigmoid(b); z: [T, H, d_k], b: [T, H]."""
    z, b, A_log = _f64(z), _f64(b), _f64(A_log)
    T, H, dk = z.shape
    g = np.empty((T, H, dk), np.float64)
    beta = np.empty((T, H), np.float64)
    lib().gdn_oracle_kda_gates(_ptr(z), _ptr(b), _ptr(A_log), T, H, dk, _ptr(g), _ptr(beta))
    return g, beta


def kda_rule(q, k, v, g, beta, state=None, threads: int | None = None):
    """KDA recurrence over one sequence: q, k: [T, H, d_k]; v: [T, H, d_v];
    g: [T, H, d_k]; beta: [T, H]; state: [H, d_v, d_k] (None = zeros).
    Returns (o [T, H, d_v], final state)."""
    q, k, v, g, beta = _f64(q), _f64(k), _f64(v), _f64(g), _f64(beta)
    T, H, dk = k.shape
    dv = v.shape[2]
    S = np.zeros((H, dv, dk)) if state is None else _f64(state).copy()
    o = np.empty((T, H, dv), np.float64)
    lib().gdn_oracle_kda_rule(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(beta), T, H, dk, dv, _ptr(S),
                              _ptr(o), threads or default_threads())
    return o, S


def sigmoid_rmsnorm(o, gate, w, eps: float = 1e-6) -> np.ndarray:
    """y = o / sqrt(mean(o^2) + eps) * w * sigmoid(gate), over the last axis."""
    o, gate, w = _f64(o), _f64(gate), _f64(w)
    d = o.shape[-1]
    y = np.empty_like(o)
    lib().gdn_oracle_sigmoid_rmsnorm(_ptr(o), _ptr(gate), _ptr(w), o.size // d, d, eps, _ptr(y))
    return y


def kda_layer(shape: Shape, qkv, zdec, b, gate, conv_w, A_log, norm_w, state=None,
              conv_window=None, heads=None, threads: int | None = None):
    """One sequence through the KDA mixer (one q, k and v head per head).

    qkv: [T, 3 H d] pre-conv rows (q heads, k heads, v heads); zdec: [T, H, d]
    decay inputs; b: [T, H]; gate: [T, H, d]; conv_w: [3 H d, K]; A_log: [H];
    norm_w: [d]; state: [H, d, d]; conv_window: [K-1, 3 H d].  With `heads`,
    only those heads are computed (every per-head output holds just them).
    Returns y, o, state and conv_window (the last K-1 pre-conv rows).
    """
    d, H, K = shape.head_dim, shape.num_v_heads, shape.conv_kernel
    assert shape.num_qk_heads == H
    T = int(qkv.shape[0])
    heads = list(range(H)) if heads is None else list(heads)
    hv = len(heads)
    cols = np.concatenate([np.arange(h * d, (h + 1) * d) for h in heads] +
                          [H * d + np.arange(h * d, (h + 1) * d) for h in heads] +
                          [2 * H * d + np.arange(h * d, (h + 1) * d) for h in heads])
    x = _take(qkv, cols, 1)
    w = _take(conv_w, cols, 0)
    win = None if conv_window is None else _take(conv_window, cols, 1)
    xc = conv_silu(x, w, win)
    q = l2norm(xc[:, : hv * d].reshape(T, hv, d), shape.l2_eps, shape.q_scale)
    k = l2norm(xc[:, hv * d: 2 * hv * d].reshape(T, hv, d), shape.l2_eps, 1.0)
    v = xc[:, 2 * hv * d:].reshape(T, hv, d)
    g, beta = kda_gates(_take(zdec, heads, 1), _take(b, heads, 1), _take(A_log, heads, 0))
    S0 = None if state is None else _take(state, heads, 0)
    o, S = kda_rule(q, k, v, g, beta, S0, threads)
    y = sigmoid_rmsnorm(o, _take(gate, heads, 1), norm_w, shape.rms_eps)
    prev = np.zeros((K - 1, x.shape[1])) if win is None else win
    hist = np.concatenate([prev, x], axis=0)
    return {"y": y, "o": o, "state": S, "conv_window": hist[-(K - 1):].copy(), "g": g,
            "beta": beta, "q": q, "k": k, "v": v}
