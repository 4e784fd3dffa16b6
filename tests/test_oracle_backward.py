"""Pins of the float64 backward oracle (oracle/backward.py), CPU only.

The backward oracle differentiates torch restatements of the TTT-Linear and
TTT-MLP scans.  These tests tie it to things other than itself:
- its primal equals the C oracle's scan (both models);
- every gradient equals central finite differences of the C oracle (both);
- for TTT-Linear, in Theorem 1's setting (plain f, one mini-batch, W0 = 0; Key takeaways
  bullet 3 of the literature record) the gradients have a closed form, that
  of causal linear attention with per-token weights 2 eta_s.
"""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import backward as ob

PLAIN, LN = oracle.MODE_PLAIN, oracle.MODE_LN_RESIDUAL


def case(seed, T=10, d=4, mode=LN, B=1, H=1):
    r = np.random.default_rng(seed)
    Q, K, V = (r.normal(0, 1 / np.sqrt(d), (B, H, T, d)) for _ in range(3))
    eta = 1 / (1 + np.exp(-r.normal(0, 1, (B, H, T)))) / d * 4
    W0 = r.normal(0, 0.3, (B, H, d, d))
    b0 = r.normal(0, 0.1, (B, H, d)) if mode == LN else np.zeros((B, H, d))
    gamma = 1 + r.normal(0, 0.2, (H, d))
    beta = r.normal(0, 0.2, (H, d))
    dZ = r.normal(0, 1, (B, H, T, d))
    dW = r.normal(0, 1, (B, H, d, d))
    db = r.normal(0, 1, (B, H, d))
    return Q, K, V, eta, W0, b0, gamma, beta, dZ, dW, db


def rel(a, b):
    a, b = np.asarray(a), np.asarray(b)
    return np.abs(a - b).max() / max(np.abs(b).max(), 1e-300)


@pytest.mark.parametrize("mode,mb,T", [(LN, 4, 10), (LN, 16, 24), (PLAIN, 4, 10), (LN, 1, 7), (LN, 8, 8)])
def test_torch_primal_equals_c_oracle(mode, mb, T):
    Q, K, V, eta, W0, b0, gamma, beta, *_ = case(1, T=T, mode=mode, B=2, H=2)
    Zt, Wt, bt = ob.linear_forward(Q, K, V, eta, W0, b0, gamma, beta, mb, mode)
    Zc, Wc, bc = oracle.ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, mb, mode)
    assert rel(Zt, Zc) < 1e-12
    assert rel(Wt, Wc) < 1e-12
    if mode == LN:
        assert rel(bt, bc) < 1e-12


def scalar_loss(inputs, mb, mode, dZ, dW, db):
    Z, W_T, b_T = oracle.ttt_linear(*inputs, mb, mode)
    L = float((Z * dZ).sum() + (W_T * dW).sum())
    if mode == LN:
        L += float((b_T * db).sum())
    return L


@pytest.mark.parametrize("mode,mb", [(LN, 4), (PLAIN, 4), (LN, 10)])
def test_gradients_equal_finite_differences_of_the_c_oracle(mode, mb):
    Q, K, V, eta, W0, b0, gamma, beta, dZ, dW, db = case(2, mode=mode)
    names = ["Q", "K", "V", "eta", "W0", "b0", "gamma", "beta"]
    inputs = [Q, K, V, eta, W0, b0, gamma, beta]
    grads = ob.ttt_linear_backward(Q, K, V, eta, W0, b0, gamma, beta, dZ, mb, mode, dW_T=dW, db_T=db)
    h = 1e-6
    for i, (name, x) in enumerate(zip(names, inputs)):
        if mode == PLAIN and name in ("b0", "gamma", "beta"):
            assert grads[i] is None
            continue
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            j = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[j] += h
            xm[j] -= h
            ip, im = list(inputs), list(inputs)
            ip[i], im[i] = xp, xm
            fd[j] = (scalar_loss(ip, mb, mode, dZ, dW, db) - scalar_loss(im, mb, mode, dZ, dW, db)) / (2 * h)
        assert rel(grads[i], fd) < 1e-6, f"d{name}: {rel(grads[i], fd):.2e}"


def test_float32_evaluation_is_the_same_algorithm():
    """The backward oracle's single-precision evaluation (the fp32 floor that sets
    the bar for long sequences) runs the same steps: on a short, well-conditioned case
    it agrees with the float64 result to single-precision rounding, and its
    outputs are float32."""
    import torch
    Q, K, V, eta, W0, b0, gamma, beta, dZ, dW, db = case(5, T=24, d=8, B=1, H=2)
    g64 = ob.ttt_linear_backward(Q, K, V, eta, W0, b0, gamma, beta, dZ, 8, LN, dW_T=dW, db_T=db)
    g32 = ob.ttt_linear_backward(Q, K, V, eta, W0, b0, gamma, beta, dZ, 8, LN, dW_T=dW, db_T=db,
                                 dtype=torch.float32)
    for a, b in zip(g32, g64):
        assert a.dtype == np.float32
        assert rel(a, b) < 1e-4
        assert rel(a, b) > 0  # rounded, not a copy of the float64 result


def test_theorem1_gradients_closed_form():
    """Plain f, eta as given, W0 = 0 and one mini-batch over all T tokens:
    z_t = sum_{s<=t} 2 eta_s (q_t . k_s) v_s, so with upstream dZ
      dQ = (M o (dZ V^T) o E) K,  dK = (M o (dZ V^T) o E)^T Q,
      dV = (M o (Q K^T) o E)^T dZ,  deta_s = sum_{t>=s} 2 (q_t . k_s)(v_s . dz_t),
    with M the lower-triangular ones and E[t, s] = 2 eta_s; and
      dW0 = sum_t (I - 2 S_t) q_t^T dz_t,  S_t = sum_{s<=t} eta_s k_s^T k_s."""
    r = np.random.default_rng(7)
    T, d = 12, 5
    Q, K, V = (r.normal(0, 1, (1, 1, T, d)) for _ in range(3))
    eta = r.uniform(0.1, 0.6, (1, 1, T))
    dZ = r.normal(0, 1, (1, 1, T, d))
    W0 = np.zeros((1, 1, d, d))
    g = ob.ttt_linear_backward(Q, K, V, eta, W0, None, None, None, dZ, T, PLAIN)
    q, k, v, e, dz = Q[0, 0], K[0, 0], V[0, 0], eta[0, 0], dZ[0, 0]
    M = np.tril(np.ones((T, T)))
    E = 2 * e[None, :]
    A = M * (dz @ v.T) * E
    np.testing.assert_allclose(g[0][0, 0], A @ k, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[1][0, 0], A.T @ q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(g[2][0, 0], (M * (q @ k.T) * E).T @ dz, rtol=1e-12, atol=1e-12)
    deta = np.array([sum(2 * (q[t] @ k[s]) * (v[s] @ dz[t]) for t in range(s, T)) for s in range(T)])
    np.testing.assert_allclose(g[3][0, 0], deta, rtol=1e-12, atol=1e-12)
    dW0 = np.zeros((d, d))
    S = np.zeros((d, d))
    for t in range(T):
        S += e[t] * np.outer(k[t], k[t])
        dW0 += (np.eye(d) - 2 * S) @ np.outer(q[t], dz[t])
    np.testing.assert_allclose(g[4][0, 0], dW0, rtol=1e-11, atol=1e-12)


# ---------------------------------------------------------------- TTT-MLP

def mlp_case(seed, T=10, d=4, hid=6):
    r = np.random.default_rng(seed)
    Q, K, V = (r.normal(0, 1 / np.sqrt(d), (1, 1, T, d)) for _ in range(3))
    eta = 1 / (1 + np.exp(-r.normal(0, 1, (1, 1, T)))) / d * 4
    W1 = r.normal(0, 1 / np.sqrt(d), (1, 1, d, hid))
    b1 = r.normal(0, 0.1, (1, 1, hid))
    W2 = r.normal(0, 1 / np.sqrt(hid), (1, 1, hid, d))
    b2 = r.normal(0, 0.1, (1, 1, d))
    gamma = 1 + r.normal(0, 0.2, (1, d))
    beta = r.normal(0, 0.2, (1, d))
    dZ = r.normal(0, 1, (1, 1, T, d))
    dS = (r.normal(0, 1, (1, 1, d, hid)), r.normal(0, 1, (1, 1, hid)), r.normal(0, 1, (1, 1, hid, d)),
          r.normal(0, 1, (1, 1, d)))
    return [Q, K, V, eta, W1, b1, W2, b2, gamma, beta], dZ, dS


@pytest.mark.parametrize("mb,T", [(4, 10), (1, 5), (8, 8)])
def test_mlp_torch_primal_equals_c_oracle(mb, T):
    ins, _, _ = mlp_case(3, T=T)
    got = ob.mlp_forward(*ins, mb)
    ref = oracle.ttt_mlp(*ins, mb)
    for g, r in zip(got, ref):
        assert rel(g, r) < 1e-12


def test_mlp_gradients_equal_finite_differences_of_the_c_oracle():
    ins, dZ, dS = mlp_case(4)
    mb = 4
    grads = ob.ttt_mlp_backward(*ins, dZ, mb, d_state=dS)

    def loss(xs):
        out = oracle.ttt_mlp(*xs, mb)
        return float((out[0] * dZ).sum() + sum((o * w).sum() for o, w in zip(out[1:], dS)))

    names = ["Q", "K", "V", "eta", "W1", "b1", "W2", "b2", "gamma", "beta"]
    h = 1e-6
    for i, (name, x) in enumerate(zip(names, ins)):
        fd = np.zeros_like(x)
        it = np.nditer(x, flags=["multi_index"])
        for _ in it:
            j = it.multi_index
            xp, xm = x.copy(), x.copy()
            xp[j] += h
            xm[j] -= h
            ip, im = list(ins), list(ins)
            ip[i], im[i] = xp, xm
            fd[j] = (loss(ip) - loss(im)) / (2 * h)
        assert rel(grads[i], fd) < 1e-6, f"d{name}: {rel(grads[i], fd):.2e}"
