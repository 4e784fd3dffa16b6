"""Pins of the float64 oracle against what the pages and mathematics fix.

Nothing here touches the CUDA library.  Each pin is independent of the
oracle's own code: closed forms (Theorem 1), finite differences and torch
autograd for every gradient, torch's LayerNorm / GELU routines for f, the
literal online-GD rule for b = 1, and invariants (eta = 0, state
continuation).  ``test_planted_mistakes_are_caught`` checks that the pins
catch plausible mistakes by compiling mutated copies of the oracle.

Sources: literature record of "Learning to (Learn at Test Time): RNNs with
Expressive Hidden States", Key takeaways bullets 1 (update and output rule),
2 (loss), 3 (Theorem 1) and 5 (mini-batch b = 16, LayerNorm and residual).
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np
import pytest
import torch

import oracle
from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs, select_heads

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden")
F64 = torch.float64
PLAIN, LN = oracle.MODE_PLAIN, oracle.MODE_LN_RESIDUAL


def rng(seed):
    return np.random.default_rng(seed)


# ----------------------------------------------------------------------------
# Independent restatements (torch float64; LayerNorm/GELU from torch)
# ----------------------------------------------------------------------------

def t64(x):
    return torch.as_tensor(np.asarray(x, dtype=np.float64))


def f_linear(x, W, b, gamma, beta, mode, eps=1e-6):
    if mode == PLAIN:
        return x @ W
    y = x @ W + b
    return x + torch.nn.functional.layer_norm(y, (y.shape[-1],), gamma, beta, eps)


def f_mlp(x, W1, b1, W2, b2, gamma, beta, eps=1e-6):
    a = torch.nn.functional.gelu(x @ W1 + b1, approximate="tanh")
    y = a @ W2 + b2
    return x + torch.nn.functional.layer_norm(y, (y.shape[-1],), gamma, beta, eps)


def autograd_grads(fn, params, k, v):
    ps = [p.detach().clone().requires_grad_(True) for p in params]
    loss = ((fn(k, *ps) - v) ** 2).sum()
    grads = torch.autograd.grad(loss, ps, allow_unused=True)
    return loss.item(), [torch.zeros_like(p) if g is None else g.detach()
                         for p, g in zip(ps, grads)]


def minibatch_restatement(fn, params, Q, K, V, eta, mb):
    """The mini-batch rule written out: gradients at the mini-batch start state,
    W_t = W_start - sum_{s<=t in mini-batch} eta_s grad_s, z_t = f(q_t; W_t)."""
    T = Q.shape[0]
    start = [p.clone() for p in params]
    Z = torch.zeros_like(Q)
    for m in range(0, T, mb):
        cur = [p.clone() for p in start]
        for t in range(m, min(m + mb, T)):
            _, gs = autograd_grads(fn, start, K[t], V[t])
            cur = [c - eta[t] * g for c, g in zip(cur, gs)]
            Z[t] = fn(Q[t], *cur)
        start = cur
    return Z, start


def small_linear_case(seed, T=48, d=8, mode=LN, w_std=0.3):
    r = rng(seed)
    Q, K, V = (r.normal(0, 1 / np.sqrt(d), (1, 1, T, d)) for _ in range(3))
    eta = 1 / (1 + np.exp(-r.normal(0, 1, (1, 1, T)))) / d * 4
    W0 = r.normal(0, w_std, (1, 1, d, d))
    b0 = r.normal(0, 0.1, (1, 1, d)) if mode == LN else np.zeros((1, 1, d))
    gamma = 1 + r.normal(0, 0.2, (1, d))
    beta = r.normal(0, 0.2, (1, d))
    return Q, K, V, eta, W0, b0, gamma, beta


def small_mlp_case(seed, T=32, d=6, hid=10):
    r = rng(seed)
    Q, K, V = (r.normal(0, 1 / np.sqrt(d), (1, 1, T, d)) for _ in range(3))
    eta = 1 / (1 + np.exp(-r.normal(0, 1, (1, 1, T)))) / d * 4
    W1 = r.normal(0, 1 / np.sqrt(d), (1, 1, d, hid))
    b1 = r.normal(0, 0.1, (1, 1, hid))
    W2 = r.normal(0, 1 / np.sqrt(hid), (1, 1, hid, d))
    b2 = r.normal(0, 0.1, (1, 1, d))
    gamma = 1 + r.normal(0, 0.2, (1, d))
    beta = r.normal(0, 0.2, (1, d))
    return Q, K, V, eta, W1, b1, W2, b2, gamma, beta


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


# ----------------------------------------------------------------------------
# Theorem 1 (Key takeaways, bullet 3)
# ----------------------------------------------------------------------------

def read_golden(name):
    vals = {}
    with open(os.path.join(GOLDEN, name)) as fh:
        for line in fh:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *nums = line.split()
            vals[key] = np.array([float(x) for x in nums])
    return vals


def test_theorem1_worked_example():
    g = read_golden("theorem1_worked_example.txt")
    T, d = 3, 2
    K = g["K"].reshape(1, 1, T, d)
    V = g["V"].reshape(1, 1, T, d)
    Q = g["Q"].reshape(1, 1, T, d)
    eta = np.full((1, 1, T), 0.5)
    Z, W_T, _ = oracle.ttt_linear(Q, K, V, eta, np.zeros((1, 1, d, d)), None, None, None,
                                  mini_batch=T, mode=PLAIN)
    np.testing.assert_array_equal(Z.reshape(-1), g["Z"])
    np.testing.assert_array_equal(W_T.reshape(-1), g["W_T"])


def test_theorem1_closed_form_full_config():
    """Theorem-1 workload (B=2, H=4, T=1024, d=64): batch GD with eta = 1/2 and
    W0 = 0 equals causal linear attention sum_{s<=t} (Q_t . K_s) V_s."""
    w = WORKLOADS["theorem1_f32"]
    inp = make_inputs(w, 0)
    Z, W_T, _ = oracle.ttt_linear(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"], None,
                                  None, None, w.mini_batch, PLAIN)
    Q, K, V = (inp[k].double() for k in "QKV")
    S = torch.tril(Q @ K.transpose(-1, -2))
    Zref = (S @ V).numpy()
    assert rel(Z, Zref) < 1e-12
    W_ref = (K.transpose(-1, -2) @ V).numpy()  # sum_s K_s^T V_s
    assert rel(W_T, W_ref) < 1e-12


# ----------------------------------------------------------------------------
# Gradients (Key takeaways, bullet 2): finite differences and autograd
# ----------------------------------------------------------------------------

def central_diff(loss_fn, x, h):
    g = np.zeros_like(x)
    it = np.nditer(x, flags=["multi_index"])
    for _ in it:
        i = it.multi_index
        xp, xm = x.copy(), x.copy()
        xp[i] += h
        xm[i] -= h
        g[i] = (loss_fn(xp) - loss_fn(xm)) / (2 * h)
    return g


@pytest.mark.parametrize("mode", [LN, PLAIN])
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_linear_gradient_finite_differences(mode, seed):
    d = 6
    r = rng(seed)
    k, v = r.normal(0, 0.5, d), r.normal(0, 0.5, d)
    W, b = r.normal(0, 0.3, (d, d)), r.normal(0, 0.1, d)
    gamma, beta = 1 + r.normal(0, 0.2, d), r.normal(0, 0.2, d)
    _, gW, gb = oracle.linear_loss_grad(k, v, W, b, gamma, beta, mode)
    fW = lambda W_: oracle.linear_loss_grad(k, v, W_, b, gamma, beta, mode)[0]
    fb = lambda b_: oracle.linear_loss_grad(k, v, W, b_, gamma, beta, mode)[0]
    h = 1e-6
    assert rel(gW, central_diff(fW, W, h)) < 1e-7
    if mode == LN:
        assert rel(gb, central_diff(fb, b, h)) < 1e-7


@pytest.mark.parametrize("mode", [LN, PLAIN])
def test_linear_gradient_autograd(mode):
    d = 8
    r = rng(7)
    k, v = r.normal(0, 0.5, d), r.normal(0, 0.5, d)
    W, b = r.normal(0, 0.05, (d, d)), r.normal(0, 0.02, d)
    gamma, beta = 1 + r.normal(0, 0.2, d), r.normal(0, 0.2, d)
    loss, gW, gb = oracle.linear_loss_grad(k, v, W, b, gamma, beta, mode)
    fn = lambda x, W_, b_: f_linear(x, W_, b_, t64(gamma), t64(beta), mode)
    loss_ref, (gW_ref, gb_ref) = autograd_grads(fn, [t64(W), t64(b)], t64(k), t64(v))
    assert abs(loss - loss_ref) <= 1e-12 * abs(loss_ref)
    assert rel(gW, gW_ref) < 1e-11
    if mode == LN:
        assert rel(gb, gb_ref) < 1e-11


@pytest.mark.parametrize("seed", [0, 1])
def test_mlp_gradient_finite_differences(seed):
    d, hid = 5, 7
    r = rng(seed)
    k, v = r.normal(0, 0.5, d), r.normal(0, 0.5, d)
    W1, b1 = r.normal(0, 0.6, (d, hid)), r.normal(0, 0.2, hid)
    W2, b2 = r.normal(0, 0.4, (hid, d)), r.normal(0, 0.2, d)
    gamma, beta = 1 + r.normal(0, 0.2, d), r.normal(0, 0.2, d)
    args = [k, v, W1, b1, W2, b2, gamma, beta]
    _, gW1, gb1, gW2, gb2 = oracle.mlp_loss_grad(*args)
    h = 1e-6
    for idx, g in ((2, gW1), (3, gb1), (4, gW2), (5, gb2)):
        def fn(x, idx=idx):
            a = list(args)
            a[idx] = x
            return oracle.mlp_loss_grad(*a)[0]
        assert rel(g, central_diff(fn, args[idx], h)) < 1e-7


def test_mlp_gradient_autograd():
    d, hid = 6, 12
    r = rng(3)
    k, v = r.normal(0, 0.5, d), r.normal(0, 0.5, d)
    W1, b1 = r.normal(0, 0.6, (d, hid)), r.normal(0, 0.2, hid)
    W2, b2 = r.normal(0, 0.4, (hid, d)), r.normal(0, 0.2, d)
    gamma, beta = 1 + r.normal(0, 0.2, d), r.normal(0, 0.2, d)
    loss, *grads = oracle.mlp_loss_grad(k, v, W1, b1, W2, b2, gamma, beta)
    fn = lambda x, a, b_, c, e: f_mlp(x, a, b_, c, e, t64(gamma), t64(beta))
    loss_ref, grads_ref = autograd_grads(fn, [t64(W1), t64(b1), t64(W2), t64(b2)], t64(k),
                                         t64(v))
    assert abs(loss - loss_ref) <= 1e-12 * abs(loss_ref)
    for g, gr in zip(grads, grads_ref):
        assert rel(g, gr) < 1e-11


# ----------------------------------------------------------------------------
# Update rule and mini-batch semantics (bullets 1 and 5)
# ----------------------------------------------------------------------------

@pytest.mark.parametrize("mode", [LN, PLAIN])
def test_b1_equals_online_gd(mode):
    """b = 1: W_t = W_{t-1} - eta_t grad l(W_{t-1}; x_t), z_t = f(q_t; W_t)."""
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(11, T=40, mode=mode)
    Z, W_T, b_T = oracle.ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, 1, mode)
    g, bt = t64(gamma[0]), t64(beta[0])
    fn = lambda x, W_, b_: f_linear(x, W_, b_, g, bt, mode)
    W, b = t64(W0[0, 0]), t64(b0[0, 0])
    Qt, Kt, Vt = t64(Q[0, 0]), t64(K[0, 0]), t64(V[0, 0])
    Zref = torch.zeros_like(Qt)
    for t in range(Qt.shape[0]):
        _, (gW, gb) = autograd_grads(fn, [W, b], Kt[t], Vt[t])
        W = W - eta[0, 0, t] * gW
        b = b - eta[0, 0, t] * gb
        Zref[t] = fn(Qt[t], W, b)
    assert rel(Z[0, 0], Zref.numpy()) < 1e-11
    assert rel(W_T[0, 0], W.numpy()) < 1e-11


@pytest.mark.parametrize("mode,mb,T", [(LN, 8, 48), (LN, 16, 48), (PLAIN, 8, 48), (LN, 48, 48),
                                       (LN, 16, 43), (PLAIN, 16, 21)])
def test_minibatch_rule_linear(mode, mb, T):
    """Includes ragged T: the last mini-batch holds the remaining T mod b tokens."""
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(5, T=T, mode=mode)
    Z, W_T, b_T = oracle.ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, mb, mode)
    g, bt = t64(gamma[0]), t64(beta[0])
    fn = lambda x, W_, b_: f_linear(x, W_, b_, g, bt, mode)
    Zref, (W_ref, b_ref) = minibatch_restatement(
        fn, [t64(W0[0, 0]), t64(b0[0, 0])], t64(Q[0, 0]), t64(K[0, 0]), t64(V[0, 0]),
        eta[0, 0], mb)
    assert rel(Z[0, 0], Zref.numpy()) < 1e-11
    assert rel(W_T[0, 0], W_ref.numpy()) < 1e-11
    if mode == LN:
        assert rel(b_T[0, 0], b_ref.numpy()) < 1e-11


@pytest.mark.parametrize("mb,T", [(1, 24), (8, 24), (16, 27)])
def test_minibatch_rule_mlp(mb, T):
    Q, K, V, eta, W1, b1, W2, b2, gamma, beta = small_mlp_case(9, T=T)
    Z, W1_T, b1_T, W2_T, b2_T = oracle.ttt_mlp(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, mb)
    g, bt = t64(gamma[0]), t64(beta[0])
    fn = lambda x, a, b_, c, e: f_mlp(x, a, b_, c, e, g, bt)
    Zref, finals = minibatch_restatement(
        fn, [t64(W1[0, 0]), t64(b1[0, 0]), t64(W2[0, 0]), t64(b2[0, 0])], t64(Q[0, 0]),
        t64(K[0, 0]), t64(V[0, 0]), eta[0, 0], mb)
    assert rel(Z[0, 0], Zref.numpy()) < 1e-11
    for got, ref in zip((W1_T, b1_T, W2_T, b2_T), finals):
        assert rel(got[0, 0], ref.numpy()) < 1e-11


def test_batch_gd_b_equals_T_ln_mode():
    """b = T: every gradient at W0 (batch GD, the setting of Theorem 1) with LN/residual."""
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(21, T=32)
    Z, W_T, b_T = oracle.ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, 32, LN)
    g, bt = t64(gamma[0]), t64(beta[0])
    W, b = t64(W0[0, 0]).requires_grad_(True), t64(b0[0, 0]).requires_grad_(True)
    Kt, Vt, Qt = t64(K[0, 0]), t64(V[0, 0]), t64(Q[0, 0])
    e = t64(eta[0, 0])
    # per-token gradients at W0, vectorised: dl_t/dy_t from one backward of sum_t l_t
    y = Kt @ W + b
    f = Kt + torch.nn.functional.layer_norm(y, (y.shape[-1],), g, bt, 1e-6)
    gy, = torch.autograd.grad(((f - Vt) ** 2).sum(), y)
    Wt = W.detach() - torch.cumsum(e[:, None, None] * Kt[:, :, None] * gy[:, None, :], 0)
    bt_ = b.detach() - torch.cumsum(e[:, None] * gy, 0)
    yq = torch.einsum("ti,tij->tj", Qt, Wt) + bt_
    Zref = Qt + torch.nn.functional.layer_norm(yq, (yq.shape[-1],), g, bt, 1e-6)
    assert rel(Z[0, 0], Zref.numpy()) < 1e-11
    assert rel(W_T[0, 0], Wt[-1].numpy()) < 1e-11


# ----------------------------------------------------------------------------
# Special cases and invariants
# ----------------------------------------------------------------------------

def test_eta_zero_linear_is_f_at_W0():
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(4, T=32)
    Z, W_T, b_T = oracle.ttt_linear(Q, K, V, np.zeros_like(eta), W0, b0, gamma, beta, 16, LN)
    Zref = f_linear(t64(Q[0, 0]), t64(W0[0, 0]), t64(b0[0, 0]), t64(gamma[0]), t64(beta[0]), LN)
    assert rel(Z[0, 0], Zref.numpy()) < 1e-13
    np.testing.assert_array_equal(W_T, W0)
    np.testing.assert_array_equal(b_T, b0)


def test_eta_zero_mlp_is_f_at_W0():
    """With eta = 0 the output is f(q; W0): LayerNorm and the tanh-form GELU from torch."""
    Q, K, V, eta, W1, b1, W2, b2, gamma, beta = small_mlp_case(6)
    Z, W1_T, b1_T, W2_T, b2_T = oracle.ttt_mlp(Q, K, V, np.zeros_like(eta), W1, b1, W2, b2,
                                               gamma, beta, 8)
    Zref = f_mlp(t64(Q[0, 0]), t64(W1[0, 0]), t64(b1[0, 0]), t64(W2[0, 0]), t64(b2[0, 0]),
                 t64(gamma[0]), t64(beta[0]))
    assert rel(Z[0, 0], Zref.numpy()) < 1e-13
    np.testing.assert_array_equal(W1_T, W1)
    np.testing.assert_array_equal(W2_T, W2)


@pytest.mark.parametrize("kind", ["linear", "mlp"])
def test_state_continuation(kind):
    """Running [0, T/2) then [T/2, T) from the carried state equals one run."""
    if kind == "linear":
        Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(8, T=64)
        full = oracle.ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, 16, LN)
        h = 32
        a = oracle.ttt_linear(Q[:, :, :h], K[:, :, :h], V[:, :, :h], eta[:, :, :h], W0, b0,
                              gamma, beta, 16, LN)
        b = oracle.ttt_linear(Q[:, :, h:], K[:, :, h:], V[:, :, h:], eta[:, :, h:], a[1], a[2],
                              gamma, beta, 16, LN)
        np.testing.assert_array_equal(np.concatenate([a[0], b[0]], axis=2), full[0])
        np.testing.assert_array_equal(b[1], full[1])
        np.testing.assert_array_equal(b[2], full[2])
    else:
        Q, K, V, eta, W1, b1, W2, b2, gamma, beta = small_mlp_case(8, T=32)
        full = oracle.ttt_mlp(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, 8)
        h = 16
        a = oracle.ttt_mlp(Q[:, :, :h], K[:, :, :h], V[:, :, :h], eta[:, :, :h], W1, b1, W2, b2,
                           gamma, beta, 8)
        b = oracle.ttt_mlp(Q[:, :, h:], K[:, :, h:], V[:, :, h:], eta[:, :, h:], *a[1:], gamma,
                           beta, 8)
        np.testing.assert_array_equal(np.concatenate([a[0], b[0]], axis=2), full[0])
        for x, y in zip(b[1:], full[1:]):
            np.testing.assert_array_equal(x, y)


def test_heads_are_independent():
    """Every (b, h) scan is independent: a gathered subset reproduces its rows exactly."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=3, T=64)
    inp = make_inputs(w, 1)
    full = oracle.ttt_linear(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"], inp["b0"],
                             inp["gamma"], inp["beta"], 16)
    pairs = [(1, 2), (0, 1)]
    sel = select_heads(inp, pairs)
    sub = oracle.ttt_linear(sel["Q"], sel["K"], sel["V"], sel["eta"], sel["W0"], sel["b0"],
                            sel["gamma"], sel["beta"], 16)
    for i, (b, h) in enumerate(pairs):
        np.testing.assert_array_equal(sub[0][0, i], full[0][b, h])
        np.testing.assert_array_equal(sub[1][0, i], full[1][b, h])


# ----------------------------------------------------------------------------
# The chunked dual form (the algebra the CUDA kernels use) equals the primal
# ----------------------------------------------------------------------------

def dual_form_linear(Q, K, V, eta, W0, b0, gamma, beta, mb, chunk=16, eps=1e-6):
    """Per chunk of 16 tokens: G = dl/dy for all tokens at the mini-batch start
    state (autograd), Zbar = Q W_cur + b_cur - tril(eta_s (q_t . k_s + 1)) G,
    then W_cur -= K^T diag(eta) G.  No per-token state is formed."""
    Q, K, V, W_s, b_s, g, bt = (t64(x) for x in (Q, K, V, W0, b0, gamma, beta))
    e = t64(eta)
    W_c, b_c = W_s.clone(), b_s.clone()
    Z = torch.zeros_like(Q)
    d = Q.shape[-1]
    for c0 in range(0, Q.shape[0], chunk):
        if c0 % mb == 0:
            W_s, b_s = W_c.clone(), b_c.clone()
        sl = slice(c0, c0 + chunk)
        X = K[sl]
        y = (X @ W_s + b_s).requires_grad_(True)
        f = X + torch.nn.functional.layer_norm(y, (d,), g, bt, eps)
        G, = torch.autograd.grad(((f - V[sl]) ** 2).sum(), y)
        A = torch.tril(e[sl][None, :] * (Q[sl] @ X.T + 1))
        zbar = Q[sl] @ W_c + b_c - A @ G
        Z[sl] = Q[sl] + torch.nn.functional.layer_norm(zbar, (d,), g, bt, eps)
        W_c = W_c - X.T @ (e[sl][:, None] * G)
        b_c = b_c - (e[sl][:, None] * G).sum(0)
    return Z.numpy(), W_c.numpy(), b_c.numpy()


@pytest.mark.parametrize("mb", [16, 32, 64])
def test_dual_form_equals_primal(mb):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=1, T=128)
    inp = make_inputs(w, 2)
    Z, W_T, b_T = oracle.ttt_linear(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"],
                                    inp["b0"], inp["gamma"], inp["beta"], mb)
    Zd, Wd, bd = dual_form_linear(inp["Q"][0, 0].double(), inp["K"][0, 0].double(),
                                  inp["V"][0, 0].double(), inp["eta"][0, 0], inp["W0"][0, 0],
                                  inp["b0"][0, 0], inp["gamma"][0], inp["beta"][0], mb)
    assert rel(Z[0, 0], Zd) < 1e-10
    assert rel(W_T[0, 0], Wd) < 1e-10
    assert rel(b_T[0, 0], bd) < 1e-10


# ----------------------------------------------------------------------------
# Rounding growth: the single-precision instantiation stays inside the bound
# ----------------------------------------------------------------------------

def test_float32_rounding_growth_is_inside_tolerance():
    """The same loops in float32 stay within 3e-3 RMS(Z) of float64 on the
    1.3B-layer recipe (2 heads, T = 4096): an fp32-state design can meet the bound."""
    w = WORKLOADS["linear_1p3b_32k"].with_shape(B=1, H=2, T=4096)
    inp = make_inputs(w, 0)
    args = [inp[k] for k in ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")]
    Z64, W64, _ = oracle.ttt_linear(*args, 16)
    Z32, W32, _ = oracle.ttt_linear(*args, 16, precision="f32")
    rms = np.sqrt((Z64 ** 2).mean())
    assert np.abs(Z32 - Z64).max() < 3e-3 * rms
    assert np.abs(W32 - W64).max() < 3e-3 * np.sqrt((W64 ** 2).mean())


# ----------------------------------------------------------------------------
# Regression fixture written by tests/golden/make_golden.py (oracle only)
# ----------------------------------------------------------------------------

def test_golden_regression_mlp_small():
    g = read_golden("mlp_small_seed0.txt")
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=1, T=48)
    inp = make_inputs(w, 0)
    keys = ("Q", "K", "V", "eta", "W1_0", "b1_0", "W2_0", "b2_0", "gamma", "beta")
    Z, W1_T, b1_T, W2_T, b2_T = oracle.ttt_mlp(*(inp[k] for k in keys), w.mini_batch, w.ln_eps)
    idx = g["Z_index"].astype(int)
    np.testing.assert_allclose(Z.reshape(-1)[idx], g["Z"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(W2_T.reshape(-1)[:32], g["W2_T_head"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(b1_T.reshape(-1)[:16], g["b1_T_head"], rtol=1e-12, atol=1e-14)


def test_golden_regression_linear_decode_pieces():
    g = read_golden("linear_decode_pieces_seed0.txt")
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=1, T=40)
    inp = make_inputs(w, 0)
    cuts = [int(c) for c in g["cuts"]]
    Z, _, _, W_mb, _ = decode_in_pieces(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"], inp["b0"],
                                        inp["gamma"], inp["beta"], 16, cuts)
    idx = g["Z_index"].astype(int)
    np.testing.assert_allclose(Z.reshape(-1)[idx], g["Z"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(W_mb.reshape(-1)[:32], g["W_mb_head"], rtol=1e-12, atol=1e-14)


def test_golden_regression_linear_tiny():
    g = read_golden("linear_tiny_f32_seed0.txt")
    w = WORKLOADS["linear_tiny_f32"]
    inp = make_inputs(w, 0)
    Z, W_T, b_T = oracle.ttt_linear(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"],
                                    inp["b0"], inp["gamma"], inp["beta"], w.mini_batch)
    idx = g["Z_index"].astype(int)
    np.testing.assert_allclose(Z.reshape(-1)[idx], g["Z"], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(W_T.reshape(-1)[:32], g["W_T_head"], rtol=1e-12, atol=1e-14)


# ----------------------------------------------------------------------------
# Decode: the scan continued from the middle of a mini-batch (Key takeaways,
# bullets 1 and 5), state carried between calls
# ----------------------------------------------------------------------------

def decode_in_pieces(Q, K, V, eta, W0, b0, gamma, beta, mb, cuts, mode=LN):
    """Run the oracle's decode over [0, T) in the pieces given by `cuts`,
    carrying (W, b, W_mb, b_mb) from call to call."""
    T = Q.shape[2]
    W, b, W_mb, b_mb = W0, b0, None, None
    Zs = []
    bounds = [0, *cuts, T]
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = (slice(None), slice(None), slice(a, c))
        Z, W, b, W_mb, b_mb = oracle.ttt_linear_decode(Q[sl], K[sl], V[sl], eta[sl], W, b, W_mb, b_mb,
                                                       gamma, beta, mb, a % mb, mode)
        Zs.append(Z)
    return np.concatenate(Zs, axis=2), W, b, W_mb, b_mb


@pytest.mark.parametrize("mode,mb,cuts", [
    (LN, 16, [5, 6, 21, 40]),   # ragged pieces, several inside one mini-batch
    (LN, 8, [1, 2, 3, 19, 33]),
    (LN, 48, [7, 30]),          # one mini-batch for the whole stream
    (PLAIN, 16, [3, 17, 18]),
    (LN, 1, [4, 9]),            # b = 1: online GD
])
def test_decode_pieces_equal_minibatch_rule(mode, mb, cuts):
    """Decode calls split anywhere reproduce the mini-batch rule written out with
    torch autograd over the whole stream."""
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(3, T=48, mode=mode)
    Z, W, b, _, _ = decode_in_pieces(Q, K, V, eta, W0, b0, gamma, beta, mb, cuts, mode)
    fn = (lambda x, W_, b_: f_linear(x, W_, b_, t64(gamma[0]), t64(beta[0]), mode))
    Zr, (Wr, br) = minibatch_restatement(fn, [t64(W0[0, 0]), t64(b0[0, 0])], t64(Q[0, 0]),
                                         t64(K[0, 0]), t64(V[0, 0]), t64(eta[0, 0]), mb)
    assert rel(Z[0, 0], Zr.numpy()) < 1e-11
    assert rel(W[0, 0], Wr.numpy()) < 1e-11
    if mode == LN:
        assert rel(b[0, 0], br.numpy()) < 1e-11


def test_decode_single_tokens_theorem1():
    """Token-by-token decode in plain mode, one mini-batch over the whole stream,
    eta = 1/2, W0 = 0: z_t = sum_{s<=t} (q_t . k_s) v_s (Theorem 1), and the
    mini-batch start state stays at W0 until the stream's mini-batch ends."""
    r = rng(11)
    T, d = 24, 8
    Q, K, V = (r.normal(0, 1, (1, 1, T, d)) for _ in range(3))
    eta = np.full((1, 1, T), 0.5)
    W, W_mb = np.zeros((1, 1, d, d)), None
    Z = np.zeros((1, 1, T, d))
    for t in range(T):
        sl = (slice(None), slice(None), slice(t, t + 1))
        Z[sl], W, _, W_mb, _ = oracle.ttt_linear_decode(Q[sl], K[sl], V[sl], eta[sl], W, None, W_mb, None,
                                                        None, None, T, t, PLAIN)
        if t < T - 1:
            assert not np.any(W_mb)
    S = np.tril(Q[0, 0] @ K[0, 0].T)
    assert rel(Z[0, 0], S @ V[0, 0]) < 1e-12
    assert rel(W_mb[0, 0], K[0, 0].T @ V[0, 0]) < 1e-12  # the next mini-batch starts from W_T


def test_decode_empty_call_keeps_state():
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(4, T=8)
    Wm = W0 + 0.25
    e = (slice(None), slice(None), slice(0, 0))
    Z, W, b, W_mb, b_mb = oracle.ttt_linear_decode(Q[e], K[e], V[e], eta[e], W0, b0, Wm, b0 * 2,
                                                   gamma, beta, 16, 5)
    assert Z.shape == (1, 1, 0, 8)
    np.testing.assert_array_equal(W, W0)
    np.testing.assert_array_equal(W_mb, Wm)  # mid-mini-batch: its start state is kept
    np.testing.assert_array_equal(b_mb, b0 * 2)
    _, W, _, W_mb, _ = oracle.ttt_linear_decode(Q[e], K[e], V[e], eta[e], W0, b0, Wm, b0, gamma, beta, 16, 0)
    np.testing.assert_array_equal(W_mb, W0)  # at a boundary the next mini-batch starts from W


@pytest.mark.parametrize("pos0", [-1, 16])
def test_decode_rejects_bad_position(pos0):
    Q, K, V, eta, W0, b0, gamma, beta = small_linear_case(4, T=8)
    with pytest.raises(ValueError):
        oracle.ttt_linear_decode(Q, K, V, eta, W0, b0, W0, b0, gamma, beta, 16, pos0)


@pytest.mark.parametrize("mb,cuts", [(8, [1, 2, 3, 13, 21]), (16, [5, 6, 21]), (1, [4, 9]), (32, [7, 30])])
def test_mlp_decode_pieces_equal_minibatch_rule(mb, cuts):
    """TTT-MLP decode calls cut anywhere reproduce the mini-batch rule written out
    with torch autograd over the whole stream."""
    Q, K, V, eta, W1, b1, W2, b2, gamma, beta = small_mlp_case(5, T=32)
    T = Q.shape[2]
    state = [W1, b1, W2, b2]
    start = [None] * 4
    Zs = []
    bounds = [0, *cuts, T]
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = (slice(None), slice(None), slice(a, c))
        out = oracle.ttt_mlp_decode(Q[sl], K[sl], V[sl], eta[sl], *state, *start, gamma, beta, mb, a % mb)
        Zs.append(out[0])
        state, start = list(out[1:5]), list(out[5:9])
    fn = (lambda x, W1_, b1_, W2_, b2_: f_mlp(x, W1_, b1_, W2_, b2_, t64(gamma[0]), t64(beta[0])))
    Zr, params = minibatch_restatement(fn, [t64(p[0, 0]) for p in (W1, b1, W2, b2)], t64(Q[0, 0]),
                                       t64(K[0, 0]), t64(V[0, 0]), t64(eta[0, 0]), mb)
    assert rel(np.concatenate(Zs, axis=2)[0, 0], Zr.numpy()) < 1e-11
    for got, ref in zip(state, params):
        assert rel(got[0, 0], ref.numpy()) < 1e-11


def test_mlp_decode_whole_stream_is_the_forward_scan():
    Q, K, V, eta, W1, b1, W2, b2, gamma, beta = small_mlp_case(6, T=40)
    dec = oracle.ttt_mlp_decode(Q, K, V, eta, W1, b1, W2, b2, None, None, None, None, gamma, beta, 16, 0)
    fwd = oracle.ttt_mlp(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, 16)
    for a, b in zip(dec[:5], fwd):
        np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------------------
# The pins catch plausible mistakes (mutations planted in a copy of the oracle)
# ----------------------------------------------------------------------------

MUTATIONS = {
    "drop_mean_term": ("g[j] = s * (g[j] - mean_gx - xhat[j] * mean_gxx);",
                       "g[j] = s * (g[j] - xhat[j] * mean_gxx);"),
    "drop_projection_term": ("g[j] = s * (g[j] - mean_gx - xhat[j] * mean_gxx);",
                             "g[j] = s * (g[j] - mean_gx);"),
    "wrong_update_sign": ("for (int j = 0; j < d; j++) Wi[j] -= ek * g[j];",
                          "for (int j = 0; j < d; j++) Wi[j] += ek * g[j];"),
    "gradient_at_running_state": (
        "FN(linear_token_dy)(d, mode, eps, K + row, V + row, Ws, bs, gam, bet, g, scratch);",
        "FN(linear_token_dy)(d, mode, eps, K + row, V + row, Wc, bc, gam, bet, g, scratch);"),
    "transposed_weight": ("for (int j = 0; j < dout; j++) y[j] += xi * Wi[j];",
                          "for (int j = 0; j < dout; j++) y[j] += xi * W[(long)j * din + i];"),
    "loss_scale_half": ("g[j] = 2 * r;", "g[j] = r;"),
    "no_residual": ("REAL r = x[j] + gamma[j] * xhat[j] + beta[j] - v[j];",
                    "REAL r = gamma[j] * xhat[j] + beta[j] - v[j];"),
    "unbiased_variance": ("v /= (REAL)d;", "v /= (REAL)(d - 1);"),
    "gelu_derivative_missing_term": (
        "(REAL)0.5 * x * ((REAL)1 - th * th) * c * ((REAL)1 + (REAL)3 * (REAL)0.044715 * x * x);",
        "(REAL)0.5 * x * ((REAL)1 - th * th) * c;"),
    "mlp_bias_not_updated": ("for (int j = 0; j < hid; j++) b1c[j] -= e * g1[j];", ""),
    "decode_gradient_at_running_state": (
        "FN(linear_token_dy)(d, mode, eps, K + row, V + row, Wm, bm, gam, bet, g, scratch);",
        "FN(linear_token_dy)(d, mode, eps, K + row, V + row, Wc, bc, gam, bet, g, scratch);"),
    "mlp_decode_gradient_at_running_state": (
        "FN(mlp_token_grads)(d, hid, eps, K + row, V + row, W1m, b1m, W2m, b2m, gam, bet, a, g1, g2,",
        "FN(mlp_token_grads)(d, hid, eps, K + row, V + row, W1c, b1c, W2c, b2c, gam, bet, a, g1, g2,"),
    "decode_no_minibatch_restart": (
        "if ((pos0 + t) % mb == 0) { /* a mini-batch starts at this token */",
        "if (0) {"),
}


def _build_mutant(tmpdir, name):
    src_dir = os.path.dirname(oracle.__file__)
    for f in ("ttt_oracle.c", "ttt_oracle_impl.h"):
        shutil.copy(os.path.join(src_dir, f), tmpdir)
    path = os.path.join(tmpdir, "ttt_oracle_impl.h")
    text = open(path).read()
    old, new = MUTATIONS[name]
    assert text.count(old) >= 1, f"mutation anchor for {name} not found"
    open(path, "w").write(text.replace(old, new))
    lib = os.path.join(tmpdir, f"libmut_{name}.so")
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp",
                    "-ffp-contract=off", "-o", lib, os.path.join(tmpdir, "ttt_oracle.c"), "-lm"],
                   check=True)
    return lib


def _run_pins_with(lib_path):
    """Run a representative subset of the pins against another build; return
    the number that fail."""
    saved = oracle._lib
    lib = ctypes.CDLL(lib_path)
    oracle._lib = None
    real_load = oracle._load

    def load_mutant():
        oracle._lib = None
        orig = oracle._build.build
        oracle._build.build = lambda force=False: lib_path
        try:
            return real_load()
        finally:
            oracle._build.build = orig

    oracle._lib = load_mutant()
    failures = 0
    pins = [
        test_theorem1_worked_example,
        lambda: test_linear_gradient_finite_differences(LN, 0),
        lambda: test_linear_gradient_finite_differences(PLAIN, 0),
        lambda: test_linear_gradient_autograd(LN),
        lambda: test_mlp_gradient_autograd(),
        lambda: test_mlp_gradient_finite_differences(0),
        lambda: test_b1_equals_online_gd(LN),
        lambda: test_minibatch_rule_linear(LN, 8, 48),
        lambda: test_minibatch_rule_mlp(8, 24),
        lambda: test_decode_pieces_equal_minibatch_rule(LN, 8, [1, 2, 3, 19, 33]),
        test_decode_single_tokens_theorem1,
        lambda: test_mlp_decode_pieces_equal_minibatch_rule(8, [1, 2, 3, 13, 21]),
    ]
    try:
        for pin in pins:
            try:
                pin()
            except AssertionError:
                failures += 1
    finally:
        oracle._lib = saved
        del lib
    return failures


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, tmp_path):
    lib = _build_mutant(str(tmp_path), name)
    assert _run_pins_with(lib) >= 1, f"no pin caught the planted mistake {name}"
