"""Pins of the oracle's KDA stages (the per-channel-decay variant of "Inkling vs
Kimi K3", component table, linear-attention and output-gate rows) against facts
that do not come from the KDA code itself: the Gated DeltaNet oracle it must
reduce to when every channel decays alike, the matrix form of the update on
tiny inputs, closed forms of the gates and of a one-dimensional state, and the
pure-decay and recall properties of the delta rule.
"""
import numpy as np
from scipy.special import expit

import oracle

rng = np.random.default_rng(2024)


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_kda_gates_closed_forms():
    """g = -5 sigmoid(e^A z): -2.5 at z = 0, within (-5, 0), saturating at the ends; beta = sigmoid(b)."""
    T, H, d = 3, 2, 5
    A_log = np.array([0.3, -1.2])
    z = rng.standard_normal((T, H, d))
    z[0] = 0.0
    b = rng.standard_normal((T, H))
    g, beta = oracle.kda_gates(z, b, A_log)
    np.testing.assert_array_equal(g[0], -2.5)
    np.testing.assert_allclose(g, -5.0 * expit(np.exp(A_log)[None, :, None] * z), rtol=1e-14)
    assert np.all(g < 0) and np.all(g > -5)
    np.testing.assert_allclose(beta, expit(b), rtol=1e-15)
    gs, _ = oracle.kda_gates(np.full((1, 1, 2), [60.0, -60.0]), np.zeros((1, 1)), np.zeros(1))
    np.testing.assert_allclose(gs[0, 0], [-5.0, 0.0], atol=1e-20)


def test_kda_matrix_definition_brute_force():
    """Token by token against S_t = S_{t-1} Diag(e^g) (I - beta k k^T) + beta v k^T, o_t = S_t q_t."""
    T, H, dk, dv = 7, 2, 3, 4
    q, k = rng.standard_normal((T, H, dk)), _unit(rng.standard_normal((T, H, dk)))
    v = rng.standard_normal((T, H, dv))
    g = -rng.random((T, H, dk)) * 2
    beta = rng.random((T, H))
    S0 = rng.standard_normal((H, dv, dk))
    o, S = oracle.kda_rule(q, k, v, g, beta, S0)
    for h in range(H):
        M = S0[h].copy()
        for t in range(T):
            kk = k[t, h][:, None]
            M = M @ np.diag(np.exp(g[t, h])) @ (np.eye(dk) - beta[t, h] * kk @ kk.T) \
                + beta[t, h] * v[t, h][:, None] @ kk.T
            np.testing.assert_allclose(o[t, h], M @ q[t, h], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[h], M, rtol=1e-12, atol=1e-12)


def test_kda_equal_channel_decay_is_the_gated_delta_rule():
    """With the same log-decay on every key channel, KDA is the Gated DeltaNet rule."""
    T, H, d = 11, 3, 6
    q, k = rng.standard_normal((T, H, d)), _unit(rng.standard_normal((T, H, d)))
    v = rng.standard_normal((T, H, d))
    g1 = -rng.random((T, H)) * 3
    beta = rng.random((T, H))
    S0 = rng.standard_normal((H, d, d))
    o_k, S_k = oracle.kda_rule(q, k, v, np.repeat(g1[:, :, None], d, axis=2), beta, S0)
    o_g, S_g = oracle.delta_rule(q, k, v, g1, beta, S0)
    np.testing.assert_allclose(o_k, o_g, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S_k, S_g, rtol=1e-12, atol=1e-12)


def test_kda_pure_decay_scales_columns():
    """beta = 0: nothing is written; column c of the state decays by exp(sum_t g_t[c])."""
    T, H, d = 9, 2, 5
    q, k = rng.standard_normal((T, H, d)), _unit(rng.standard_normal((T, H, d)))
    v = rng.standard_normal((T, H, d))
    g = -rng.random((T, H, d))
    S0 = rng.standard_normal((H, d, d))
    o, S = oracle.kda_rule(q, k, v, g, np.zeros((T, H)), S0)
    decay = np.exp(np.cumsum(g, axis=0))  # [T, H, d]
    for t in range(T):
        for h in range(H):
            St = S0[h] * decay[t, h][None, :]
            np.testing.assert_allclose(o[t, h], St @ q[t, h], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, S0 * decay[-1][:, None, :], rtol=1e-12, atol=1e-13)


def test_kda_write_recalls_value():
    """beta = 1 with a unit key: after the step, S_t k_t = v_t exactly, whatever the decay."""
    T, H, d = 6, 1, 4
    q, k = rng.standard_normal((T, H, d)), _unit(rng.standard_normal((T, H, d)))
    v = rng.standard_normal((T, H, d))
    g = -rng.random((T, H, d)) * 2
    S0 = rng.standard_normal((H, d, d))
    for t in range(1, T + 1):
        _, S = oracle.kda_rule(q[:t], k[:t], v[:t], g[:t], np.ones((t, H)), S0)
        np.testing.assert_allclose(S[0] @ k[t - 1, 0], v[t - 1, 0], rtol=1e-12, atol=1e-12)


def test_kda_scalar_closed_form():
    """d = 1, k = +-1: s_t = e^{g_t} (1 - beta_t) s_{t-1} + beta_t v_t k_t, o_t = s_t q_t."""
    T = 12
    q = rng.standard_normal((T, 1, 1))
    k = np.sign(rng.standard_normal((T, 1, 1)))
    v = rng.standard_normal((T, 1, 1))
    g = -rng.random((T, 1, 1))
    beta = rng.random((T, 1))
    o, S = oracle.kda_rule(q, k, v, g, beta, np.array([[[0.7]]]))
    s = 0.7
    for t in range(T):
        s = np.exp(g[t, 0, 0]) * (1 - beta[t, 0]) * s + beta[t, 0] * v[t, 0, 0] * k[t, 0, 0]
        np.testing.assert_allclose(o[t, 0, 0], s * q[t, 0, 0], rtol=1e-13)
    np.testing.assert_allclose(S[0, 0, 0], s, rtol=1e-13)


def test_sigmoid_rmsnorm():
    """y / (w sigmoid(gate)) has unit mean square (eps aside); the gate is the logistic function."""
    rows, d = 6, 16
    o = rng.standard_normal((rows, d)) * 3
    gate = rng.standard_normal((rows, d))
    w = 1 + 0.1 * rng.standard_normal(d)
    y = oracle.sigmoid_rmsnorm(o, gate, w, eps=0.0)
    base = y / (w[None] * expit(gate))
    np.testing.assert_allclose(np.mean(base ** 2, axis=1), 1.0, rtol=1e-12)
    np.testing.assert_allclose(base, o / np.sqrt(np.mean(o ** 2, axis=1, keepdims=True)), rtol=1e-12)


def _kda_inputs(T, H=2, d=8, seed=3):
    r = np.random.default_rng(seed)
    C = 3 * H * d
    return dict(qkv=r.standard_normal((T, C)), zdec=r.standard_normal((T, H, d)),
                b=r.standard_normal((T, H)), gate=r.standard_normal((T, H, d)),
                conv_w=0.5 * r.standard_normal((C, 4)), A_log=np.log(r.uniform(1, 16, H)),
                norm_w=1 + 0.1 * r.standard_normal(d)), oracle.Shape(H, H, d)


def test_kda_layer_decode_and_split_equal_whole():
    """Prefill T then one more token (with the carried state and conv window) and a
    split prefill both equal the prefill of the whole sequence."""
    x, shape = _kda_inputs(21)
    P = {k: x[k] for k in ("conv_w", "A_log", "norm_w")}
    cut = lambda s, e: {k: x[k][s:e] for k in ("qkv", "zdec", "b", "gate")}
    whole = oracle.kda_layer(shape, **cut(0, 21), **P)
    a = oracle.kda_layer(shape, **cut(0, 13), **P)
    b = oracle.kda_layer(shape, **cut(13, 20), **P, state=a["state"], conv_window=a["conv_window"])
    c = oracle.kda_layer(shape, **cut(20, 21), **P, state=b["state"], conv_window=b["conv_window"])
    np.testing.assert_allclose(np.concatenate([a["y"], b["y"], c["y"]]), whole["y"], rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(c["state"], whole["state"], rtol=1e-11, atol=1e-12)
    np.testing.assert_array_equal(c["conv_window"], whole["conv_window"])


def test_kda_layer_head_subset_equals_full():
    x, shape = _kda_inputs(15, H=3)
    P = {k: x[k] for k in ("conv_w", "A_log", "norm_w")}
    full = oracle.kda_layer(shape, x["qkv"], x["zdec"], x["b"], x["gate"], **P)
    sub = oracle.kda_layer(shape, x["qkv"], x["zdec"], x["b"], x["gate"], **P, heads=[2, 0])
    np.testing.assert_allclose(sub["y"], full["y"][:, [2, 0]], rtol=1e-13)
    np.testing.assert_allclose(sub["state"], full["state"][[2, 0]], rtol=1e-13)
