"""Float64 oracle of the TTT layer's backward (outer-loop gradients), for
TTT-Linear and (below) TTT-MLP.

TEST INFRASTRUCTURE.  Only ``tests/`` may import this module; the CUDA library
never calls it.

What it computes: for the causal TTT-Linear scan (the literature record of
"Learning to (Learn at Test Time): RNNs with Expressive Hidden States", Key
takeaways bullets 1, 2 and 5: state W, b updated per mini-batch with
gradients taken at the mini-batch start state; output z_t = f(q_t; W_t)) and
upstream gradients dZ (and optionally dW_T, db_T of the final state), the
gradients of

    L = sum(Z * dZ) + sum(W_T * dW_T) + sum(b_T * db_T)

with respect to Q, K, V, eta, W0, b0, gamma and beta.  These are the
gradients an outer training loop needs (bullet 2: the learning rate, and the
views theta_Q, theta_K, theta_V, are trained by the outer loop).

How: the primal scan written token by token in float64 torch (the same steps
as the C oracle's loop: gradient of ||f(k_t; W_s) - v_t||^2 at the mini-batch
start state, running-state update, output with the running state), with the
inner gradient computed in closed form (LayerNorm backward written out), and
torch autograd applied to the whole scan as a library primitive.  Autograd
then supplies the second-order terms (the update depends on W_s through the
LayerNorm backward).  For TTT-MLP the inner gradient itself is taken by
autograd (with its graph kept), over the same loop.
"""
from __future__ import annotations

from typing import Optional, Tuple

import numpy as np
import torch

MODE_LN_RESIDUAL = 0
MODE_PLAIN = 1


def _t(x, requires_grad=False, dtype=torch.float64):
    if x is None:
        return None
    if hasattr(x, "detach"):
        t = x.detach().to("cpu", torch.float64).clone()
    else:
        t = torch.as_tensor(np.asarray(x, dtype=np.float64)).clone()
    return t.to(dtype).requires_grad_(requires_grad)


def _inner_grad(k, v, Ws, bs, gamma, beta, mode: int, eps: float):
    """dl/dy for l = ||f(k; W_s, b_s) - v||^2, y = k W_s + b_s (batched over [B, H])."""
    if mode == MODE_PLAIN:
        y = torch.einsum("bhi,bhij->bhj", k, Ws)
        return 2.0 * (y - v)
    y = torch.einsum("bhi,bhij->bhj", k, Ws) + bs
    d = y.shape[-1]
    mu = y.mean(-1, keepdim=True)
    var = ((y - mu) ** 2).mean(-1, keepdim=True)
    s = 1.0 / torch.sqrt(var + eps)
    xhat = (y - mu) * s
    r = k + gamma * xhat + beta - v            # f(k) - v, with the residual
    gx = 2.0 * gamma * r                       # dl/dxhat
    # LayerNorm backward: dl/dy = (s / d) (d gx - sum gx - xhat sum(gx xhat))
    return (s / d) * (d * gx - gx.sum(-1, keepdim=True) - xhat * (gx * xhat).sum(-1, keepdim=True))


def _apply(q, W, b, gamma, beta, mode: int, eps: float):
    if mode == MODE_PLAIN:
        return torch.einsum("bhi,bhij->bhj", q, W)
    y = torch.einsum("bhi,bhij->bhj", q, W) + b
    mu = y.mean(-1, keepdim=True)
    var = ((y - mu) ** 2).mean(-1, keepdim=True)
    return q + gamma * (y - mu) / torch.sqrt(var + eps) + beta


def linear_scan(Q, K, V, eta, W0, b0, gamma, beta, mini_batch: int, mode: int, eps: float):
    """The primal scan in float64 torch (differentiable).  Q, K, V [B,H,T,d],
    eta [B,H,T], W0 [B,H,d,d], b0 [B,H,d], gamma / beta [H,d].
    Returns (Z, W_T, b_T)."""
    B, H, T, d = Q.shape
    g = gamma[None] if gamma is not None else None   # [1,H,d]
    be = beta[None] if beta is not None else None
    Ws, bs = W0, b0
    Zs = []
    for m in range(0, T, mini_batch):
        Wc, bc = Ws, bs
        for t in range(m, min(m + mini_batch, T)):
            k, v, q = K[:, :, t], V[:, :, t], Q[:, :, t]
            e = eta[:, :, t][..., None]
            gy = _inner_grad(k, v, Ws, bs, g, be, mode, eps)
            Wc = Wc - e[..., None] * torch.einsum("bhi,bhj->bhij", k, gy)
            if mode != MODE_PLAIN:
                bc = bc - e * gy
            Zs.append(_apply(q, Wc, bc, g, be, mode, eps))
        Ws, bs = Wc, bc
    return torch.stack(Zs, dim=2), Ws, bs


def ttt_linear_backward(Q, K, V, eta, W0, b0, gamma, beta, dZ, mini_batch: int,
                        mode: int = MODE_LN_RESIDUAL, ln_eps: float = 1e-6,
                        dW_T=None, db_T=None, dtype=torch.float64) -> Tuple[np.ndarray, ...]:
    """Gradients of sum(Z dZ) + sum(W_T dW_T) + sum(b_T db_T) with respect to
    (Q, K, V, eta, W0, b0, gamma, beta).  In plain mode b0, gamma, beta may be
    None and their gradients are returned as None.

    ``dtype=torch.float32`` evaluates the same steps in single precision: not a
    reference, but the rounding floor of any fp32 implementation of the scan's
    backward, which sets the bar for a long sequence's fp32 errors."""
    plain = mode == MODE_PLAIN
    c = lambda x, rg=False: _t(x, rg, dtype)
    Qt, Kt, Vt, et, W0t = (c(x, True) for x in (Q, K, V, eta, W0))
    B, H, T, d = Qt.shape
    b0t = c(b0 if b0 is not None else np.zeros((B, H, d)), not plain)
    gt = c(gamma, not plain) if not plain else None
    bt = c(beta, not plain) if not plain else None
    Z, W_T, b_T = linear_scan(Qt, Kt, Vt, et, W0t, b0t, gt, bt, mini_batch, mode, ln_eps)
    L = (Z * c(dZ)).sum()
    if dW_T is not None:
        L = L + (W_T * c(dW_T)).sum()
    if db_T is not None and not plain:
        L = L + (b_T * c(db_T)).sum()
    wrt = [Qt, Kt, Vt, et, W0t] + ([] if plain else [b0t, gt, bt])
    grads = torch.autograd.grad(L, wrt, allow_unused=True)
    out = [None if gr is None else gr.numpy() for gr in grads]
    if plain:
        out += [None, None, None]
    return tuple(out)


def linear_forward(Q, K, V, eta, W0, b0, gamma, beta, mini_batch: int, mode: int = MODE_LN_RESIDUAL,
                   ln_eps: float = 1e-6) -> Tuple[np.ndarray, np.ndarray, Optional[np.ndarray]]:
    """The torch primal scan's outputs (for checking it against the C oracle)."""
    with torch.no_grad():
        plain = mode == MODE_PLAIN
        Qt, Kt, Vt, et, W0t = (_t(x) for x in (Q, K, V, eta, W0))
        B, H, T, d = Qt.shape
        b0t = _t(b0 if b0 is not None else np.zeros((B, H, d)))
        Z, W_T, b_T = linear_scan(Qt, Kt, Vt, et, W0t, b0t, None if plain else _t(gamma),
                                  None if plain else _t(beta), mini_batch, mode, ln_eps)
        return Z.numpy(), W_T.numpy(), None if plain else b_T.numpy()


# ---------------------------------------------------------------- TTT-MLP
def _gelu(x):
    # tanh form, as in the forward oracle
    c = 0.7978845608028654
    return 0.5 * x * (1.0 + torch.tanh(c * (x + 0.044715 * x ** 3)))


def _ln_res(x, y, gamma, beta, eps):
    mu = y.mean(-1, keepdim=True)
    var = ((y - mu) ** 2).mean(-1, keepdim=True)
    return x + gamma * (y - mu) / torch.sqrt(var + eps) + beta


def mlp_scan(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, mini_batch: int, eps: float):
    """The TTT-MLP primal scan in float64 torch (differentiable; the inner
    gradient by autograd with create_graph, so the outer gradient sees its
    dependence on the state).  Shapes as the forward oracle's.  Returns
    (Z, W1_T, b1_T, W2_T, b2_T)."""
    B, H, T, d = Q.shape
    g, be = gamma[None], beta[None]

    def f(x, W1_, b1_, W2_, b2_):
        a = _gelu(torch.einsum("bhi,bhij->bhj", x, W1_) + b1_)
        return _ln_res(x, torch.einsum("bhi,bhij->bhj", a, W2_) + b2_, g, be, eps)

    S = [W1, b1, W2, b2]
    Zs = []
    for m in range(0, T, mini_batch):
        C = list(S)
        for t in range(m, min(m + mini_batch, T)):
            k, v, q = K[:, :, t], V[:, :, t], Q[:, :, t]
            loss = ((f(k, *S) - v) ** 2).sum()
            grads = torch.autograd.grad(loss, S, create_graph=True)
            e = eta[:, :, t]
            C = [c - (e[..., None, None] if c.dim() == 4 else e[..., None]) * gr for c, gr in zip(C, grads)]
            Zs.append(f(q, *C))
        S = C
    return (torch.stack(Zs, dim=2), *S)


def ttt_mlp_backward(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, dZ, mini_batch: int,
                     ln_eps: float = 1e-6, d_state=None):
    """Gradients of sum(Z dZ) (+ sum over the final state times d_state, a
    tuple (dW1_T, db1_T, dW2_T, db2_T)) with respect to (Q, K, V, eta, W1, b1,
    W2, b2, gamma, beta)."""
    ins = [_t(x, True) for x in (Q, K, V, eta, W1, b1, W2, b2, gamma, beta)]
    out = mlp_scan(*ins, mini_batch, ln_eps)
    L = (out[0] * _t(dZ)).sum()
    if d_state is not None:
        for s_, ds_ in zip(out[1:], d_state):
            L = L + (s_ * _t(ds_)).sum()
    return tuple(gr.numpy() for gr in torch.autograd.grad(L, ins))


def mlp_forward(Q, K, V, eta, W1, b1, W2, b2, gamma, beta, mini_batch: int, ln_eps: float = 1e-6):
    """The torch primal's outputs (for checking it against the C oracle)."""
    ins = [_t(x, True) for x in (Q, K, V, eta, W1, b1, W2, b2, gamma, beta)]
    return tuple(o.detach().numpy() for o in mlp_scan(*ins, mini_batch, ln_eps))
