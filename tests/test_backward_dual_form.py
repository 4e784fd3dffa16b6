"""The TTT layer backward (TTT-Linear, then TTT-MLP) as a backward kernel
would run it, checked against the pinned float64 backward oracle
(oracle/backward.py).  CPU only.

A restatement of the algorithm, not a second oracle.  Forward: chunk by chunk
(a chunk is one mini-batch of b <= 16 tokens) in the dual form, keeping each
chunk's start state; the states are small, 16.6 KB per chunk and head, so a
GPU keeps them all: 2.2 GB for the 64 scans of the 1.3B/32k shape.  Backward:
chunk by chunk in reverse, recomputing the chunk's intermediates from its
start state, with the adjoint of every step written out by hand.  That
includes the second-order terms through the LayerNorm backward that forms
the inner gradient G.  ("Learning to (Learn at Test Time)", literature
record, Key takeaways bullets 1, 2 and 5.)
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import backward as ob


def _ln_rows(y, eps):
    mu = y.mean(1, keepdims=True)
    s = 1.0 / np.sqrt(((y - mu) ** 2).mean(1, keepdims=True) + eps)
    return (y - mu) * s, s


def _chunk_forward(Q, X, V, e, W, b, gam, bet, eps):
    """One chunk in the dual form; returns its outputs, new state and the
    intermediates the backward reuses."""
    d = X.shape[1]
    Y = X @ W + b
    xh, s = _ln_rows(Y, eps)
    R = X + gam * xh + bet - V
    Gx = 2.0 * gam * R
    m1 = Gx.mean(1, keepdims=True)
    m2 = (Gx * xh).mean(1, keepdims=True)
    G = s * (Gx - m1 - xh * m2)
    P = Q @ X.T
    M = np.tril(np.ones((X.shape[0], X.shape[0])))
    A = M * (e[None, :] * (P + 1.0))
    Zb = Q @ W + b - A @ G
    zh, s2 = _ln_rows(Zb, eps)
    Z = Q + gam * zh + bet
    Wn = W - X.T @ (e[:, None] * G)
    bn = b - (e[:, None] * G).sum(0)
    cache = dict(Y=Y, xh=xh, s=s, R=R, Gx=Gx, m1=m1, m2=m2, G=G, P=P, M=M, A=A, zh=zh, s2=s2, d=d)
    return Z, Wn, bn, cache


def _ln_back(dxh, xh, s):
    """x^ = (y - mean y) s with s = (var y + eps)^(-1/2): dy from dx^."""
    return s * (dxh - dxh.mean(1, keepdims=True) - xh * (dxh * xh).mean(1, keepdims=True))


def dual_form_backward(Q, K, V, eta, W0, b0, gam, bet, dZ, dW_T, db_T, chunk, eps=1e-6):
    """Gradients of sum(Z dZ) + sum(W_T dW_T) + sum(b_T db_T) for one (batch,
    head): Q, K, V, dZ [T, d], eta [T], W0 [d, d], b0, gam, bet [d]; one chunk
    is one mini-batch (chunk <= 16).  Returns dQ, dK, dV, deta, dW0, db0,
    dgam, dbet."""
    T, d = Q.shape
    starts = list(range(0, T, chunk))
    states = []
    W, b = W0, b0
    for c0 in starts:
        sl = slice(c0, c0 + chunk)
        states.append((W, b))
        _, W, b, _ = _chunk_forward(Q[sl], K[sl], V[sl], eta[sl], W, b, gam, bet, eps)
    dQ, dK, dV, de = (np.zeros_like(x) for x in (Q, K, V, eta))
    dgam, dbet = np.zeros_like(gam), np.zeros_like(bet)
    dW, db = dW_T.copy(), db_T.copy()           # gradient of the state after the chunk
    for c0, (W, b) in zip(reversed(starts), reversed(states)):
        sl = slice(c0, c0 + chunk)
        Qc, X, Vc, e = Q[sl], K[sl], V[sl], eta[sl]
        _, _, _, k = _chunk_forward(Qc, X, Vc, e, W, b, gam, bet, eps)
        G, A, xh, s, zh = k["G"], k["A"], k["xh"], k["s"], k["zh"]
        # z = q + gam z^ + bet, z^ = LN(Zb)
        dz = dZ[sl]
        dgam += (dz * zh).sum(0)
        dbet += dz.sum(0)
        dQc = dz.copy()
        dZb = _ln_back(dz * gam, zh, k["s2"])
        # Zb = Q W + b - A G
        dQc += dZb @ W.T
        dW_prev = Q[sl].T @ dZb
        db_prev = dZb.sum(0)
        dA = -(dZb @ G.T) * k["M"]
        dG = -A.T @ dZb
        # W' = W - X^T diag(eta) G, b' = b - G^T eta
        dEG = -(X @ dW) - db[None, :]
        dG += e[:, None] * dEG
        de[sl] += (dEG * G).sum(1)
        dXc = -(e[:, None] * G) @ dW.T
        dW_prev += dW
        db_prev += db
        # A = tril(eta_s (P + 1)), P = Q X^T
        de[sl] += (dA * (k["P"] + 1.0)).sum(0)
        dP = dA * e[None, :]
        dQc += dP @ X
        dXc += dP.T @ Qc
        # G = s (Gx - m1 - x^ m2), Gx = 2 gam R, R = X + gam x^ + bet - V
        mdg = (dG * xh).mean(1, keepdims=True)
        dGx = s * (dG - dG.mean(1, keepdims=True)) - s * mdg * xh
        dxh = -s * k["m2"] * dG - s * mdg * k["Gx"]
        ds = (dG * (k["Gx"] - k["m1"] - xh * k["m2"])).sum(1, keepdims=True)
        dR = 2.0 * gam * dGx
        dgam += (2.0 * k["R"] * dGx).sum(0) + (dR * xh).sum(0)
        dbet += dR.sum(0)
        dXc += dR
        dV[sl] = -dR
        dxh += gam * dR
        # x^ = LN(Y) without affine; s also appears explicitly in G
        dY = _ln_back(dxh, xh, s) - ds * s * s * xh / d
        # Y = X W + b
        dXc += dY @ W.T
        dW_prev += X.T @ dY
        db_prev += dY.sum(0)
        dQ[sl], dK[sl] = dQc, dXc
        dW, db = dW_prev, db_prev
    return dQ, dK, dV, de, dW, db, dgam, dbet


def case(seed, T, d=8):
    r = np.random.default_rng(seed)
    Q, K, V = (r.normal(0, 1 / np.sqrt(d), (1, 1, T, d)) for _ in range(3))
    eta = 1 / (1 + np.exp(-r.normal(0, 1, (1, 1, T)))) / d * 4
    W0 = r.normal(0, 0.3, (1, 1, d, d))
    b0 = r.normal(0, 0.1, (1, 1, d))
    gamma = 1 + r.normal(0, 0.2, (1, d))
    beta = r.normal(0, 0.2, (1, d))
    dZ = r.normal(0, 1, (1, 1, T, d))
    dW = r.normal(0, 1, (1, 1, d, d))
    db = r.normal(0, 1, (1, 1, d))
    return Q, K, V, eta, W0, b0, gamma, beta, dZ, dW, db


def rel(a, b):
    return np.abs(np.asarray(a) - b).max() / max(np.abs(b).max(), 1e-300)


@pytest.mark.parametrize("T,chunk", [(48, 16), (40, 16), (24, 8), (7, 1), (16, 16)])
def test_chunked_backward_equals_the_oracle(T, chunk):
    Q, K, V, eta, W0, b0, gamma, beta, dZ, dW, db = case(T + chunk, T)
    ref = ob.ttt_linear_backward(Q, K, V, eta, W0, b0, gamma, beta, dZ, chunk, dW_T=dW, db_T=db)
    got = dual_form_backward(Q[0, 0], K[0, 0], V[0, 0], eta[0, 0], W0[0, 0], b0[0, 0], gamma[0], beta[0],
                             dZ[0, 0], dW[0, 0], db[0, 0], chunk)
    names = ("dQ", "dK", "dV", "deta", "dW0", "db0", "dgamma", "dbeta")
    for name, g, r in zip(names, got, ref):
        r = r[0, 0] if name not in ("dgamma", "dbeta") else r[0]
        assert rel(g, r) < 1e-10, f"{name}: {rel(g, r):.2e}"


# ---------------------------------------------------------------- TTT-MLP

_C = 0.7978845608028654  # sqrt(2 / pi)


def _gelu(x):
    return 0.5 * x * (1.0 + np.tanh(_C * (x + 0.044715 * x ** 3)))


def _gelu_d1(x):
    th = np.tanh(_C * (x + 0.044715 * x ** 3))
    du = _C * (1.0 + 3 * 0.044715 * x * x)
    return 0.5 * (1.0 + th) + 0.5 * x * (1.0 - th * th) * du


def _gelu_d2(x):
    th = np.tanh(_C * (x + 0.044715 * x ** 3))
    du = _C * (1.0 + 3 * 0.044715 * x * x)
    d2u = _C * 6 * 0.044715 * x
    return (1.0 - th * th) * (du + 0.5 * x * (d2u - 2.0 * th * du * du))


def _mlp_chunk_forward(Q, X, V, e, W1, b1, W2, b2, gam, bet, eps):
    n, d = X.shape
    M = np.tril(np.ones((n, n)))
    Z1 = X @ W1 + b1
    Hh = _gelu(Z1)
    Y = Hh @ W2 + b2
    xh, s = _ln_rows(Y, eps)
    R = X + gam * xh + bet - V
    Gx = 2.0 * gam * R
    m1 = Gx.mean(1, keepdims=True)
    m2 = (Gx * xh).mean(1, keepdims=True)
    G2 = s * (Gx - m1 - xh * m2)
    U = G2 @ W2.T
    G1 = U * _gelu_d1(Z1)
    P = Q @ X.T
    A = M * (e[None, :] * (P + 1.0))
    Z1q = Q @ W1 + b1 - A @ G1
    Hq = _gelu(Z1q)
    P2 = Hq @ Hh.T
    A2 = M * (e[None, :] * (P2 + 1.0))
    Z2q = Hq @ W2 + b2 - A2 @ G2
    zh, s2 = _ln_rows(Z2q, eps)
    Z = Q + gam * zh + bet
    new = (W1 - X.T @ (e[:, None] * G1), b1 - (e[:, None] * G1).sum(0),
           W2 - Hh.T @ (e[:, None] * G2), b2 - (e[:, None] * G2).sum(0))
    cache = dict(M=M, Z1=Z1, Hh=Hh, xh=xh, s=s, R=R, Gx=Gx, m1=m1, m2=m2, G2=G2, U=U, G1=G1, P=P, A=A,
                 Z1q=Z1q, Hq=Hq, P2=P2, A2=A2, zh=zh, s2=s2, d=d)
    return Z, new, cache


def mlp_dual_form_backward(Q, K, V, eta, W1, b1, W2, b2, gam, bet, dZ, dS, chunk, eps=1e-6):
    """TTT-MLP counterpart of dual_form_backward: gradients of sum(Z dZ) plus
    the final state times dS = (dW1_T, db1_T, dW2_T, db2_T) for one (batch,
    head).  Returns dQ, dK, dV, deta, dW1, db1, dW2, db2, dgam, dbet."""
    T, d = Q.shape
    starts = list(range(0, T, chunk))
    states, S = [], (W1, b1, W2, b2)
    for c0 in starts:
        sl = slice(c0, c0 + chunk)
        states.append(S)
        _, S, _ = _mlp_chunk_forward(Q[sl], K[sl], V[sl], eta[sl], *S, gam, bet, eps)
    dQ, dK, dV, de = (np.zeros_like(x) for x in (Q, K, V, eta))
    dgam, dbet = np.zeros_like(gam), np.zeros_like(bet)
    dW1n, db1n, dW2n, db2n = (x.copy() for x in dS)   # gradient of the state after the chunk
    for c0, (cW1, cb1, cW2, cb2) in zip(reversed(starts), reversed(states)):
        sl = slice(c0, c0 + chunk)
        Qc, X, Vc, e = Q[sl], K[sl], V[sl], eta[sl]
        _, _, k = _mlp_chunk_forward(Qc, X, Vc, e, cW1, cb1, cW2, cb2, gam, bet, eps)
        M, G1, G2, Hh, Hq = k["M"], k["G1"], k["G2"], k["Hh"], k["Hq"]
        dW1, db1, dW2, db2 = dW1n.copy(), db1n.copy(), dW2n.copy(), db2n.copy()
        # output: z = q + gam z^ + bet, z^ = LN(Z2q)
        dz = dZ[sl]
        dgam += (dz * k["zh"]).sum(0)
        dbet += dz.sum(0)
        dQc = dz.copy()
        dZ2q = _ln_back(dz * gam, k["zh"], k["s2"])
        # Z2q = Hq W2 + b2 - A2 G2
        dHq = dZ2q @ cW2.T
        dW2 += Hq.T @ dZ2q
        db2 += dZ2q.sum(0)
        dA2 = -(dZ2q @ G2.T) * M
        dG2 = -k["A2"].T @ dZ2q
        # A2 = tril(eta_s (Hq Hh^T + 1))
        de[sl] += (dA2 * (k["P2"] + 1.0)).sum(0)
        dP2 = dA2 * e[None, :]
        dHq += dP2 @ Hh
        dHh = dP2.T @ Hq
        # Hq = gelu(Z1q); Z1q = Q W1 + b1 - A G1
        dZ1q = dHq * _gelu_d1(k["Z1q"])
        dQc += dZ1q @ cW1.T
        dW1 += Qc.T @ dZ1q
        db1 += dZ1q.sum(0)
        dA = -(dZ1q @ G1.T) * M
        dG1 = -k["A"].T @ dZ1q
        # A = tril(eta_s (Q X^T + 1))
        de[sl] += (dA * (k["P"] + 1.0)).sum(0)
        dP = dA * e[None, :]
        dQc += dP @ X
        dXc = dP.T @ Qc
        # state update: W1' = W1 - X^T (eta G1), b1' = b1 - (eta G1)^T 1; the same for W2 with Hh, G2
        dE1 = -(X @ dW1n) - db1n[None, :]
        dG1 += e[:, None] * dE1
        de[sl] += (dE1 * G1).sum(1)
        dXc += -(e[:, None] * G1) @ dW1n.T
        dE2 = -(Hh @ dW2n) - db2n[None, :]
        dG2 += e[:, None] * dE2
        de[sl] += (dE2 * G2).sum(1)
        dHh += -(e[:, None] * G2) @ dW2n.T
        # G1 = (G2 W2^T) * gelu'(Z1)
        dU = dG1 * _gelu_d1(k["Z1"])
        dZ1 = dG1 * k["U"] * _gelu_d2(k["Z1"])
        dG2 += dU @ cW2
        dW2 += dU.T @ G2
        # G2 = LayerNorm backward of the reconstruction loss at Y
        xh, s = k["xh"], k["s"]
        mdg = (dG2 * xh).mean(1, keepdims=True)
        dGx = s * (dG2 - dG2.mean(1, keepdims=True)) - s * mdg * xh
        dxh = -s * k["m2"] * dG2 - s * mdg * k["Gx"]
        ds = (dG2 * (k["Gx"] - k["m1"] - xh * k["m2"])).sum(1, keepdims=True)
        dR = 2.0 * gam * dGx
        dgam += (2.0 * k["R"] * dGx).sum(0) + (dR * xh).sum(0)
        dbet += dR.sum(0)
        dXc += dR
        dV[sl] = -dR
        dxh += gam * dR
        dY = _ln_back(dxh, xh, s) - ds * s * s * xh / k["d"]
        # Y = Hh W2 + b2; Hh = gelu(Z1); Z1 = X W1 + b1
        dHh += dY @ cW2.T
        dW2 += Hh.T @ dY
        db2 += dY.sum(0)
        dZ1 += dHh * _gelu_d1(k["Z1"])
        dXc += dZ1 @ cW1.T
        dW1 += X.T @ dZ1
        db1 += dZ1.sum(0)
        dQ[sl], dK[sl] = dQc, dXc
        dW1n, db1n, dW2n, db2n = dW1, db1, dW2, db2
    return dQ, dK, dV, de, dW1n, db1n, dW2n, db2n, dgam, dbet


def mlp_case(seed, T, d=6, hid=10):
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


def test_gelu_derivatives_against_differences():
    x = np.linspace(-4, 4, 81)
    h = 1e-5
    assert rel(_gelu_d1(x), (_gelu(x + h) - _gelu(x - h)) / (2 * h)) < 1e-8
    assert rel(_gelu_d2(x), (_gelu_d1(x + h) - _gelu_d1(x - h)) / (2 * h)) < 1e-7


@pytest.mark.parametrize("T,chunk", [(24, 8), (20, 8), (12, 4), (5, 1)])
def test_mlp_chunked_backward_equals_the_oracle(T, chunk):
    ins, dZ, dS = mlp_case(T + chunk, T)
    ref = ob.ttt_mlp_backward(*ins, dZ, chunk, d_state=dS)
    squeeze = lambda x: x[0, 0] if x.ndim >= 3 else x[0]
    got = mlp_dual_form_backward(*(squeeze(x) for x in ins), squeeze(dZ), tuple(squeeze(x) for x in dS), chunk)
    names = ("dQ", "dK", "dV", "deta", "dW1", "db1", "dW2", "db2", "dgamma", "dbeta")
    for name, g, r in zip(names, got, ref):
        assert rel(g, squeeze(r)) < 1e-10, f"{name}: {rel(g, squeeze(r)):.2e}"
