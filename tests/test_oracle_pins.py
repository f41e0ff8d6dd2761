"""Pins of the FP64 oracle against facts that do not come from the oracle itself.

Each test fixes one stage (or the whole layer) by a closed form, a library
routine, an invariant of the mathematics, or brute force on tiny inputs, so
that a plausible slip in the oracle (a reversed conv tap, a decay applied
after the write instead of before, a transposed state, a wrong q/k-head
mapping, a norm over the wrong axis, the gate applied before the norm) fails
at least one of them.
"""
import math

import numpy as np
import pytest
from scipy.special import expit

import oracle

rng = np.random.default_rng(12345)


# ------------------------------------------------------------------ conv


def test_conv_matches_numpy_convolve():
    """Causal kernel-4 depthwise conv == np.convolve with the taps reversed, first T outputs."""
    T, C, K = 23, 5, 4
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, K))
    # pre-activation: undo SiLU by comparing silu(reference) with the oracle output
    out = oracle.conv_silu(x, w)
    for c in range(C):
        ref = np.convolve(x[:, c], w[c, ::-1])[:T]
        np.testing.assert_allclose(out[:, c], ref * expit(ref), rtol=1e-13, atol=1e-14)


def test_conv_window_equals_prepending_rows():
    """A conv window of K-1 rows behaves exactly like those rows placed before the sequence."""
    T, C, K = 9, 4, 4
    x = rng.standard_normal((T, C))
    win = rng.standard_normal((K - 1, C))
    w = rng.standard_normal((C, K))
    with_win = oracle.conv_silu(x, w, win)
    full = oracle.conv_silu(np.concatenate([win, x]), w)
    np.testing.assert_allclose(with_win, full[K - 1:], rtol=0, atol=1e-15)


def test_conv_causal_and_kernel_support():
    """Perturbing token t changes outputs t..t+3 only (causality + kernel size 4)."""
    T, C = 16, 3
    x = rng.standard_normal((T, C))
    w = rng.standard_normal((C, 4)) + 0.5
    base = oracle.conv_silu(x, w)
    t = 6
    x2 = x.copy()
    x2[t] += 1.0
    pert = oracle.conv_silu(x2, w)
    changed = np.any(np.abs(pert - base) > 0, axis=1)
    assert not changed[:t].any()
    assert changed[t:t + 4].all()
    assert not changed[t + 4:].any()


def test_silu_via_identity_conv():
    """With taps (0,0,0,1) the stage is SiLU alone: x * sigmoid(x) from scipy."""
    x = np.linspace(-30, 30, 61).reshape(61, 1)
    w = np.array([[0.0, 0.0, 0.0, 1.0]])
    np.testing.assert_allclose(oracle.conv_silu(x, w)[:, 0], x[:, 0] * expit(x[:, 0]),
                               rtol=1e-14, atol=1e-300)
    assert oracle.conv_silu(np.zeros((1, 1)), w)[0, 0] == 0.0


# ---------------------------------------------------------------- l2norm


def test_l2norm_unit_length_and_direction():
    x = rng.standard_normal((7, 3, 32)) * 5
    y = oracle.l2norm(x, eps=0.0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), 1.0, rtol=0, atol=1e-14)
    # parallel to the input, per row of the last axis (not over another axis)
    cos = np.sum(x * y, -1) / np.linalg.norm(x, axis=-1)
    np.testing.assert_allclose(cos, 1.0, atol=1e-14)
    y2 = oracle.l2norm(x, eps=0.0, scale=0.25)
    np.testing.assert_allclose(y2, 0.25 * y, rtol=1e-15)


def test_l2norm_eps_inside_sqrt():
    x = np.full((1, 4), 0.5)  # sum of squares = 1
    y = oracle.l2norm(x, eps=3.0)
    np.testing.assert_allclose(y, 0.5 / 2.0, rtol=1e-15)


# ----------------------------------------------------------------- gates


def test_gates_closed_forms():
    A_log = np.log(np.array([1.0, 2.0, 16.0]))
    dt_bias = np.array([0.3, -1.2, 2.0])
    # a + dt_bias = 0  ->  softplus = ln 2  ->  g = -exp(A_log) ln 2 ; b = 0 -> beta = 1/2
    a = -dt_bias[None, :].copy()
    b = np.zeros((1, 3))
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    np.testing.assert_allclose(g[0], -np.exp(A_log) * math.log(2.0), rtol=1e-15)
    np.testing.assert_allclose(beta[0], 0.5, rtol=0)
    # general points against numpy's logaddexp (softplus) and scipy's expit (sigmoid)
    a = rng.standard_normal((50, 3)) * 20
    b = rng.standard_normal((50, 3)) * 20
    g, beta = oracle.gates(a, b, A_log, dt_bias)
    np.testing.assert_allclose(g, -np.exp(A_log) * np.logaddexp(0.0, a + dt_bias), rtol=1e-14)
    np.testing.assert_allclose(beta, expit(b), rtol=1e-14)
    assert np.all(g < 0) and np.all((beta > 0) & (beta <= 1))


# ------------------------------------------------------------ delta rule


def _unit(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


def test_delta_rule_matrix_definition_brute_force():
    """Token by token against S_t = a_t S_{t-1} (I - b_t k k^T) + b_t v k^T, o_t = S_t q_t."""
    T, Hk, Hv, dk, dv = 11, 1, 2, 3, 4
    q = rng.standard_normal((T, Hk, dk))
    k = _unit(rng.standard_normal((T, Hk, dk)))
    v = rng.standard_normal((T, Hv, dv))
    g = -rng.random((T, Hv)) * 2
    beta = rng.random((T, Hv))
    S0 = rng.standard_normal((Hv, dv, dk))
    o, S = oracle.delta_rule(q, k, v, g, beta, S0, threads=1)
    for h in range(Hv):
        St = S0[h].copy()
        for t in range(T):
            kk = k[t, 0][:, None]
            St = math.exp(g[t, h]) * St @ (np.eye(dk) - beta[t, h] * kk @ kk.T) \
                + beta[t, h] * v[t, h][:, None] @ kk.T
            np.testing.assert_allclose(o[t, h], St @ q[t, 0], rtol=1e-12, atol=1e-12)
        np.testing.assert_allclose(S[h], St, rtol=1e-12, atol=1e-12)


def test_delta_rule_write_recalls_value():
    """beta = 1 with unit keys: right after token t, S_t k_t = v_t exactly."""
    T, d = 20, 8
    q = _unit(rng.standard_normal((T, 1, d)))
    k = _unit(rng.standard_normal((T, 1, d)))
    v = rng.standard_normal((T, 1, d))
    g = -rng.random((T, 1))
    beta = np.ones((T, 1))
    for t_end in (1, 5, T):
        _, S = oracle.delta_rule(q[:t_end], k[:t_end], v[:t_end], g[:t_end], beta[:t_end],
                                 rng.standard_normal((1, d, d)))
        np.testing.assert_allclose(S[0] @ k[t_end - 1, 0], v[t_end - 1, 0], atol=1e-12)


def test_delta_rule_identity_step():
    """beta = 0 and g = 0 leave the state unchanged and read o = S0 q."""
    T, d = 6, 5
    q = rng.standard_normal((T, 1, d))
    k = _unit(rng.standard_normal((T, 1, d)))
    v = rng.standard_normal((T, 1, d))
    S0 = rng.standard_normal((1, d, d))
    o, S = oracle.delta_rule(q, k, v, np.zeros((T, 1)), np.zeros((T, 1)), S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o[:, 0], q[:, 0] @ S0[0].T, rtol=1e-14)


def test_delta_rule_reset_by_large_decay():
    """g = -1e4 (alpha underflows to 0) forgets the past: S = beta v k^T."""
    d = 6
    q = rng.standard_normal((3, 1, d))
    k = _unit(rng.standard_normal((3, 1, d)))
    v = rng.standard_normal((3, 1, d))
    beta = np.array([[0.3], [0.9], [0.7]])
    g = np.array([[-0.1], [-0.2], [-1e4]])
    _, S = oracle.delta_rule(q, k, v, g, beta, rng.standard_normal((1, d, d)))
    np.testing.assert_allclose(S[0], 0.7 * np.outer(v[2, 0], k[2, 0]), atol=1e-15)


def test_delta_rule_orthogonal_keys_is_gated_linear_attention():
    """Distinct one-hot keys never interfere, so with S0 = 0
    o_t = sum_{s<=t} (prod_{r=s+1..t} alpha_r) beta_s (k_s . q_t) v_s  and
    S_T = sum_s (prod_{r=s+1..T} alpha_r) beta_s v_s k_s^T."""
    d = 12
    T = d
    q = rng.standard_normal((T, 1, d))
    k = np.eye(d)[rng.permutation(d)][:, None, :]
    v = rng.standard_normal((T, 1, d))
    g = -rng.random((T, 1)) * 1.5
    beta = rng.random((T, 1))
    o, S = oracle.delta_rule(q, k, v, g, beta)
    alpha = np.exp(g[:, 0])
    for t in range(T):
        ref = np.zeros(d)
        for s in range(t + 1):
            ref += np.prod(alpha[s + 1:t + 1]) * beta[s, 0] * (k[s, 0] @ q[t, 0]) * v[s, 0]
        np.testing.assert_allclose(o[t, 0], ref, rtol=1e-12, atol=1e-14)
    Sref = sum(np.prod(alpha[s + 1:]) * beta[s, 0] * np.outer(v[s, 0], k[s, 0]) for s in range(T))
    np.testing.assert_allclose(S[0], Sref, rtol=1e-12, atol=1e-14)


def test_delta_rule_scalar_closed_form():
    """d = 1, k = +-1: s_t = alpha_t (1 - beta_t) s_{t-1} + beta_t v_t k_t, o_t = s_t q_t."""
    T = 40
    k = rng.choice([-1.0, 1.0], size=(T, 1, 1))
    q = rng.standard_normal((T, 1, 1))
    v = rng.standard_normal((T, 1, 1))
    g = -rng.random((T, 1))
    beta = rng.random((T, 1))
    o, S = oracle.delta_rule(q, k, v, g, beta, np.array([[[0.7]]]))
    s = 0.7
    for t in range(T):
        s = math.exp(g[t, 0]) * (1 - beta[t, 0]) * s + beta[t, 0] * v[t, 0, 0] * k[t, 0, 0]
        assert abs(o[t, 0, 0] - s * q[t, 0, 0]) < 1e-13
    assert abs(S[0, 0, 0] - s) < 1e-13


def test_delta_rule_superposition():
    """o and S are jointly linear in (v, S0) for fixed q, k, g, beta."""
    T, d = 9, 6
    q = rng.standard_normal((T, 1, d))
    k = _unit(rng.standard_normal((T, 1, d)))
    g = -rng.random((T, 2))
    beta = rng.random((T, 2))
    v1, v2 = rng.standard_normal((2, T, 2, d))
    S1, S2 = rng.standard_normal((2, 2, d, d))
    o1, F1 = oracle.delta_rule(q, k, v1, g, beta, S1)
    o2, F2 = oracle.delta_rule(q, k, v2, g, beta, S2)
    o3, F3 = oracle.delta_rule(q, k, 2 * v1 - 3 * v2, g, beta, 2 * S1 - 3 * S2)
    np.testing.assert_allclose(o3, 2 * o1 - 3 * o2, atol=1e-12)
    np.testing.assert_allclose(F3, 2 * F1 - 3 * F2, atol=1e-12)


def test_delta_rule_head_mapping():
    """Value head h reads q/k head h // G: grouped run == each head run alone on its group's q, k."""
    T, Hk, G, d = 7, 3, 2, 4
    Hv = Hk * G
    q = rng.standard_normal((T, Hk, d))
    k = _unit(rng.standard_normal((T, Hk, d)))
    v = rng.standard_normal((T, Hv, d))
    g = -rng.random((T, Hv))
    beta = rng.random((T, Hv))
    S0 = rng.standard_normal((Hv, d, d))
    o, S = oracle.delta_rule(q, k, v, g, beta, S0)
    for h in range(Hv):
        j = h // G
        o1, S1 = oracle.delta_rule(q[:, j:j + 1], k[:, j:j + 1], v[:, h:h + 1], g[:, h:h + 1],
                                   beta[:, h:h + 1], S0[h:h + 1], threads=1)
        np.testing.assert_array_equal(o[:, h], o1[:, 0])
        np.testing.assert_array_equal(S[h], S1[0])
    # and perturbing q/k head 1 changes exactly value heads 2 and 3
    k2 = k.copy()
    k2[:, 1] = _unit(rng.standard_normal((T, d)))
    o2, _ = oracle.delta_rule(q, k2, v, g, beta, S0)
    diff = np.abs(o2 - o).max(axis=(0, 2))
    assert list(np.nonzero(diff > 0)[0]) == [2, 3]


# ----------------------------------------------------------- gated norm


def test_gated_rmsnorm_properties():
    R, d = 10, 32
    o = rng.standard_normal((R, d)) * 3
    z = rng.standard_normal((R, d))
    w = 1 + 0.1 * rng.standard_normal(d)
    y = oracle.gated_rmsnorm(o, z, w, eps=0.0)
    # normalised first, then gated: y / (w * silu(z)) has unit mean square per row
    n = y / (w * z * expit(z))
    np.testing.assert_allclose(np.mean(n ** 2, axis=1), 1.0, rtol=1e-13)
    np.testing.assert_allclose(n, o / np.sqrt(np.mean(o ** 2, axis=1, keepdims=True)), rtol=1e-12)
    # scale-free in o (eps = 0), and eps sits inside the root beside the mean
    np.testing.assert_allclose(oracle.gated_rmsnorm(7.5 * o, z, w, eps=0.0), y, rtol=1e-13)
    ones = np.ones((1, 4))
    big = np.full((1, 4), 40.0)  # silu(40) = 40 to double precision
    np.testing.assert_allclose(oracle.gated_rmsnorm(ones, big, np.ones(4), eps=3.0),
                               1.0 / 2.0 * 40.0, rtol=1e-15)


# ------------------------------------------------------------ whole layer


def _layer_inputs(shape, T, seed, dtype=np.float64):
    r = np.random.default_rng(seed)
    d, Hv = shape.head_dim, shape.num_v_heads
    return dict(qkv=r.standard_normal((T, shape.conv_dim)), a=r.standard_normal((T, Hv)),
                b=r.standard_normal((T, Hv)), z=r.standard_normal((T, Hv, d)),
                conv_w=r.standard_normal((shape.conv_dim, 4)) * 0.5,
                A_log=np.log(r.uniform(1, 16, Hv)), dt_bias=r.standard_normal(Hv) * 0.5,
                norm_w=1 + 0.1 * r.standard_normal(d))


SMALL = oracle.Shape(num_qk_heads=2, num_v_heads=4, head_dim=8)


def _run(shape, inp, s, e, state=None, win=None):
    p = {k: inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")}
    return oracle.layer(shape, inp["qkv"][s:e], inp["a"][s:e], inp["b"][s:e], inp["z"][s:e],
                        state=state, conv_window=win, **p)


def test_layer_prefill_then_decode_equals_longer_prefill():
    T = 13
    inp = _layer_inputs(SMALL, T + 1, 7)
    S0 = np.random.default_rng(1).standard_normal((4, 8, 8)) * 0.02
    whole = _run(SMALL, inp, 0, T + 1, S0)
    head = _run(SMALL, inp, 0, T, S0)
    p = {k: inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")}
    dec = oracle.decode(SMALL, inp["qkv"][T:T + 1], inp["a"][T:T + 1], inp["b"][T:T + 1],
                        inp["z"][T:T + 1], state=head["state"][None],
                        conv_cache=head["conv_window"][None], **p)
    np.testing.assert_allclose(dec["y"][0], whole["y"][T], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(dec["state"][0], whole["state"], rtol=1e-12, atol=1e-14)
    np.testing.assert_array_equal(dec["conv_window"][0], whole["conv_window"])
    np.testing.assert_array_equal(whole["conv_window"], inp["qkv"][T - 2:T + 1])


def test_layer_split_prefill_equals_whole():
    T, T1 = 21, 8
    inp = _layer_inputs(SMALL, T, 8)
    whole = _run(SMALL, inp, 0, T)
    a = _run(SMALL, inp, 0, T1)
    b = _run(SMALL, inp, T1, T, a["state"], a["conv_window"])
    np.testing.assert_allclose(np.concatenate([a["y"], b["y"]]), whole["y"], rtol=1e-12,
                               atol=1e-13)
    np.testing.assert_allclose(b["state"], whole["state"], rtol=1e-12, atol=1e-14)


def test_layer_packed_varlen_equals_each_alone():
    lens = [5, 1, 0, 9]
    cu = np.concatenate([[0], np.cumsum(lens)])
    inp = _layer_inputs(SMALL, int(cu[-1]), 9)
    S0 = np.random.default_rng(2).standard_normal((4, 4, 8, 8)) * 0.02
    p = {k: inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")}
    out = oracle.prefill(SMALL, inp["qkv"], inp["a"], inp["b"], inp["z"], cu,
                         initial_state=S0, **p)
    for n in range(len(lens)):
        s, e = cu[n], cu[n + 1]
        r = _run(SMALL, inp, s, e, S0[n])
        np.testing.assert_array_equal(out["y"][s:e], r["y"])
        np.testing.assert_array_equal(out["state"][n], r["state"])
    # an empty sequence passes its state through untouched, conv window stays zero
    np.testing.assert_array_equal(out["state"][2], S0[2])
    np.testing.assert_array_equal(out["conv_window"][2], 0.0)


def test_layer_group_subset_equals_full():
    """Computing one q/k group's value heads alone gives the same numbers as the full layer."""
    shape = oracle.Shape(num_qk_heads=2, num_v_heads=8, head_dim=8)
    inp = _layer_inputs(shape, 10, 10)
    S0 = np.random.default_rng(3).standard_normal((8, 8, 8))
    full = _run(shape, inp, 0, 10, S0)
    p = {k: inp[k] for k in ("conv_w", "A_log", "dt_bias", "norm_w")}
    sub = oracle.layer(shape, inp["qkv"], inp["a"], inp["b"], inp["z"], state=S0, group=1,
                       heads=[5, 7], **p)
    np.testing.assert_allclose(sub["y"], full["y"][:, [5, 7]], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(sub["state"], full["state"][[5, 7]], rtol=1e-13, atol=1e-15)


def test_layer_row_permutation_equivariance():
    """Permuting the value channels of every head (v, S0 rows, z, norm weight) permutes y and S."""
    shape = SMALL
    d = shape.head_dim
    inp = _layer_inputs(shape, 6, 11)
    S0 = np.random.default_rng(4).standard_normal((4, d, d))
    base = _run(shape, inp, 0, 6, S0)
    perm = np.random.default_rng(5).permutation(d)
    inp2 = dict(inp)
    vcols = 2 * shape.num_qk_heads * d + np.arange(shape.num_v_heads * d)
    vperm = (vcols.reshape(-1, d)[:, perm]).reshape(-1)
    qkv2 = inp["qkv"].copy()
    qkv2[:, vcols] = inp["qkv"][:, vperm]
    cw2 = inp["conv_w"].copy()
    cw2[vcols] = inp["conv_w"][vperm]
    inp2.update(qkv=qkv2, conv_w=cw2, z=inp["z"][:, :, perm], norm_w=inp["norm_w"][perm])
    out = _run(shape, inp2, 0, 6, S0[:, perm, :])
    np.testing.assert_allclose(out["y"], base["y"][:, :, perm], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(out["state"], base["state"][:, perm, :], rtol=1e-13, atol=1e-15)
