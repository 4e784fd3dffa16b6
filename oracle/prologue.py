"""Float64 oracle of the TTT layer's prologue: the per-head projections of the
layer input into the scan's Q, K, V, the token-dependent learning rate eta,
and rotary position embedding of Q and K.

TEST INFRASTRUCTURE.  Only ``tests/`` may import this module; the CUDA library
never calls it.

What the pages fix (the literature record of "Learning to (Learn at Test
Time): RNNs with Expressive Hidden States", Key takeaways bullets 1 and 2):
- the scan sees three linear views of each token, theta_K x_t (training
  input), theta_V x_t (label) and theta_Q x_t (test input);
- the learning rate is token-dependent and trained by the outer loop.
The codewithpapers.app record names the rotary helpers (rotate_half) among
the official code's entry points, without their formulas.

Readings taken where the pages are silent (each listed in the design notes):
- per head h: Q = x theta_Q[h], K = x theta_K[h], V = x theta_V[h], no bias;
- eta_t = eta_base * sigmoid(x_t . theta_lr[h] + b_lr[h]) / d;
- rotary embedding in the rotate-half convention on Q and K: feature i and
  i + d/2 rotate together by angle p * base^(-2i/d), base 10000, with p the
  token's absolute position in the sequence.
"""
from __future__ import annotations

import numpy as np


def _f64(x):
    if hasattr(x, "detach"):
        import torch
        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def rope_angles(T: int, d: int, base: float = 10000.0, pos0: int = 0) -> np.ndarray:
    """[T, d/2] rotation angles: position (pos0 + t) times base^(-2i/d)."""
    i = np.arange(d // 2, dtype=np.float64)
    inv = base ** (-2.0 * i / d)
    p = np.arange(pos0, pos0 + T, dtype=np.float64)
    return p[:, None] * inv[None, :]


def rope(x, base: float = 10000.0, pos0: int = 0) -> np.ndarray:
    """Rotate-half rotary embedding of x [..., T, d] (d even)."""
    x = _f64(x)
    T, d = x.shape[-2], x.shape[-1]
    a = rope_angles(T, d, base, pos0)
    c, s = np.cos(a), np.sin(a)
    x1, x2 = x[..., : d // 2], x[..., d // 2:]
    return np.concatenate([x1 * c - x2 * s, x2 * c + x1 * s], axis=-1)


def project(x, theta_q, theta_k, theta_v, theta_lr, b_lr, eta_base: float = 1.0, rotary: bool = True,
            base: float = 10000.0, pos0: int = 0):
    """x [B, T, D]; theta_q / theta_k / theta_v [H, D, d]; theta_lr [H, D];
    b_lr [H].  Returns Q, K, V [B, H, T, d] and eta [B, H, T] (float64)."""
    x = _f64(x)
    tq, tk, tv, tl, bl = (_f64(t) for t in (theta_q, theta_k, theta_v, theta_lr, b_lr))
    d = tq.shape[-1]
    Q = np.einsum("btD,hDd->bhtd", x, tq)
    K = np.einsum("btD,hDd->bhtd", x, tk)
    V = np.einsum("btD,hDd->bhtd", x, tv)
    logit = np.einsum("btD,hD->bht", x, tl) + bl[None, :, None]
    eta = eta_base / (1.0 + np.exp(-logit)) / d
    if rotary:
        Q, K = rope(Q, base, pos0), rope(K, base, pos0)
    return Q, K, V, eta
