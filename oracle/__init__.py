"""Float64 CPU oracle of the TTT forward scan (ctypes wrapper over plain C).

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  The CUDA library
never calls it, and it never calls the CUDA library.

Every array argument is a numpy array (or anything ``np.asarray`` accepts,
including CPU torch tensors, which are upcast exactly).  Shapes follow the
library's: Q, K, V [B,H,T,d]; eta [B,H,T]; W0 [B,H,d,d] (W[in][out]);
b0 [B,H,d]; gamma, beta [H,d]; MLP W1 [B,H,d,hid], W2 [B,H,hid,d].

Sources are cited in ``ttt_oracle_impl.h``: the literature record of
"Learning to (Learn at Test Time): RNNs with Expressive Hidden States",
Key takeaways bullets 1 (state/update/output rule), 2 (inner loss),
3 (Theorem 1) and 5 (mini-batch b = 16, LayerNorm and residual in f), and the
paper's abstract (TTT-Linear and TTT-MLP).
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np

from . import build as _build

MODE_LN_RESIDUAL = 0
MODE_PLAIN = 1

_lib = None


def _load():
    global _lib
    if _lib is None:
        path = _build.build()
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        I = ctypes.c_int
        for sfx, real in (("_f64", ctypes.c_double), ("_f32", ctypes.c_float)):
            f = getattr(lib, "oracle_ttt_linear" + sfx)
            f.restype = I
            f.argtypes = [I, I, I, I, I, I, real] + [P] * 11 + [I]
            f = getattr(lib, "oracle_ttt_linear_decode" + sfx)
            f.restype = I
            f.argtypes = [I, I, I, I, I, I, I, real] + [P] * 11 + [I]
            f = getattr(lib, "oracle_ttt_mlp" + sfx)
            f.restype = I
            f.argtypes = [I, I, I, I, I, I, real] + [P] * 15 + [I]
            f = getattr(lib, "oracle_ttt_mlp_decode" + sfx)
            f.restype = I
            f.argtypes = [I, I, I, I, I, I, I, real] + [P] * 15 + [I]
            f = getattr(lib, "oracle_linear_loss_grad" + sfx)
            f.restype = real
            f.argtypes = [I, I, real] + [P] * 8
            f = getattr(lib, "oracle_mlp_loss_grad" + sfx)
            f.restype = real
            f.argtypes = [I, I, real] + [P] * 12
        _lib = lib
    return _lib


def _arr(x, dtype) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # torch tensor: upcast on the torch side (bf16 has no numpy dtype)
        import torch
        x = x.detach().to("cpu", torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64), dtype=dtype)


def _ptr(a: Optional[np.ndarray]):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _threads(n: Optional[int]) -> int:
    return int(n) if n else (os.cpu_count() or 1)


def ttt_linear(Q, K, V, eta, W0, b0, gamma, beta, mini_batch: int,
               mode: int = MODE_LN_RESIDUAL, ln_eps: float = 1e-6,
               precision: str = "f64", threads: Optional[int] = None):
    """Primal TTT-Linear scan.  Returns (Z [B,H,T,d], W_T [B,H,d,d], b_T [B,H,d])."""
    dt = np.float64 if precision == "f64" else np.float32
    Q, K, V, eta, W0 = (_arr(x, dt) for x in (Q, K, V, eta, W0))
    B, H, T, d = Q.shape
    b0 = _arr(b0, dt) if b0 is not None else np.zeros((B, H, d), dt)
    gamma = _arr(gamma, dt) if gamma is not None else np.ones((H, d), dt)
    beta = _arr(beta, dt) if beta is not None else np.zeros((H, d), dt)
    Z = np.zeros((B, H, T, d), dt)
    W_T = np.zeros((B, H, d, d), dt)
    b_T = np.zeros((B, H, d), dt)
    fn = getattr(_load(), "oracle_ttt_linear_" + precision)
    rc = fn(B, H, T, d, int(mini_batch), int(mode), ln_eps, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
            _ptr(W0), _ptr(b0), _ptr(gamma), _ptr(beta), _ptr(Z), _ptr(W_T), _ptr(b_T),
            _threads(threads))
    if rc != 0:
        raise ValueError("oracle_ttt_linear: bad arguments")
    return Z, W_T, b_T


def ttt_linear_decode(Q, K, V, eta, W, b, W_mb, b_mb, gamma, beta, mini_batch: int, pos0: int,
                      mode: int = MODE_LN_RESIDUAL, ln_eps: float = 1e-6,
                      precision: str = "f64", threads: Optional[int] = None):
    """TTT-Linear scan continued by T tokens from position pos0 of a mini-batch.

    W, b: running state [B,H,d,d], [B,H,d]; W_mb, b_mb: state the current
    mini-batch started from (read when pos0 > 0).  Returns (Z, W, b, W_mb,
    b_mb) after the T tokens; W_mb, b_mb are then the start state of the
    mini-batch the next token falls in.  The inputs are not modified."""
    dt = np.float64 if precision == "f64" else np.float32
    Q, K, V, eta = (_arr(x, dt) for x in (Q, K, V, eta))
    B, H, T, d = Q.shape
    W = _arr(W, dt).copy()
    W_mb = _arr(W_mb, dt).copy() if W_mb is not None else W.copy()
    b = _arr(b, dt).copy() if b is not None else np.zeros((B, H, d), dt)
    b_mb = _arr(b_mb, dt).copy() if b_mb is not None else b.copy()
    gamma = _arr(gamma, dt) if gamma is not None else np.ones((H, d), dt)
    beta = _arr(beta, dt) if beta is not None else np.zeros((H, d), dt)
    Z = np.zeros((B, H, T, d), dt)
    fn = getattr(_load(), "oracle_ttt_linear_decode_" + precision)
    rc = fn(B, H, T, d, int(mini_batch), int(pos0), int(mode), ln_eps, _ptr(Q), _ptr(K), _ptr(V),
            _ptr(eta), _ptr(W), _ptr(b), _ptr(W_mb), _ptr(b_mb), _ptr(gamma), _ptr(beta), _ptr(Z),
            _threads(threads))
    if rc != 0:
        raise ValueError("oracle_ttt_linear_decode: bad arguments")
    return Z, W, b, W_mb, b_mb


def ttt_mlp(Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, gamma, beta, mini_batch: int,
            ln_eps: float = 1e-6, precision: str = "f64", threads: Optional[int] = None):
    """Primal TTT-MLP scan.  Returns (Z, W1_T, b1_T, W2_T, b2_T)."""
    dt = np.float64 if precision == "f64" else np.float32
    Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, gamma, beta = (
        _arr(x, dt) for x in (Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, gamma, beta))
    B, H, T, d = Q.shape
    hid = W1_0.shape[-1]
    Z = np.zeros((B, H, T, d), dt)
    W1_T = np.zeros((B, H, d, hid), dt)
    b1_T = np.zeros((B, H, hid), dt)
    W2_T = np.zeros((B, H, hid, d), dt)
    b2_T = np.zeros((B, H, d), dt)
    fn = getattr(_load(), "oracle_ttt_mlp_" + precision)
    rc = fn(B, H, T, d, hid, int(mini_batch), ln_eps, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
            _ptr(W1_0), _ptr(b1_0), _ptr(W2_0), _ptr(b2_0), _ptr(gamma), _ptr(beta), _ptr(Z),
            _ptr(W1_T), _ptr(b1_T), _ptr(W2_T), _ptr(b2_T), _threads(threads))
    if rc != 0:
        raise ValueError("oracle_ttt_mlp: bad arguments")
    return Z, W1_T, b1_T, W2_T, b2_T


def ttt_mlp_decode(Q, K, V, eta, W1, b1, W2, b2, W1_mb, b1_mb, W2_mb, b2_mb, gamma, beta,
                   mini_batch: int, pos0: int, ln_eps: float = 1e-6, precision: str = "f64",
                   threads: Optional[int] = None):
    """TTT-MLP scan continued by T tokens from position pos0 of a mini-batch.

    (W1, b1, W2, b2): running state; (W1_mb, ...): the state the current
    mini-batch started from (read when pos0 > 0; None means a copy of the
    running state).  Returns (Z, W1, b1, W2, b2, W1_mb, b1_mb, W2_mb, b2_mb)
    after the T tokens.  The inputs are not modified."""
    dt = np.float64 if precision == "f64" else np.float32
    Q, K, V, eta = (_arr(x, dt) for x in (Q, K, V, eta))
    B, H, T, d = Q.shape
    run = [_arr(x, dt).copy() for x in (W1, b1, W2, b2)]
    start = [(_arr(x, dt).copy() if x is not None else r.copy()) for x, r in zip((W1_mb, b1_mb, W2_mb, b2_mb), run)]
    gamma, beta = _arr(gamma, dt), _arr(beta, dt)
    hid = run[0].shape[-1]
    Z = np.zeros((B, H, T, d), dt)
    fn = getattr(_load(), "oracle_ttt_mlp_decode_" + precision)
    rc = fn(B, H, T, d, hid, int(mini_batch), int(pos0), ln_eps, _ptr(Q), _ptr(K), _ptr(V), _ptr(eta),
            *(_ptr(x) for x in run), *(_ptr(x) for x in start), _ptr(gamma), _ptr(beta), _ptr(Z),
            _threads(threads))
    if rc != 0:
        raise ValueError("oracle_ttt_mlp_decode: bad arguments")
    return (Z, *run, *start)


def linear_loss_grad(k, v, W, b, gamma, beta, mode: int = MODE_LN_RESIDUAL,
                     ln_eps: float = 1e-6):
    """Loss of one token and its gradients (dl/dW [d,d], dl/db [d]), as the scan uses them."""
    k, v, W = (_arr(x, np.float64) for x in (k, v, W))
    d = k.shape[0]
    b = _arr(b, np.float64) if b is not None else np.zeros(d)
    gamma = _arr(gamma, np.float64) if gamma is not None else np.ones(d)
    beta = _arr(beta, np.float64) if beta is not None else np.zeros(d)
    gW = np.zeros((d, d))
    gb = np.zeros(d)
    loss = _load().oracle_linear_loss_grad_f64(d, int(mode), ln_eps, _ptr(k), _ptr(v), _ptr(W),
                                               _ptr(b), _ptr(gamma), _ptr(beta), _ptr(gW),
                                               _ptr(gb))
    return loss, gW, gb


def mlp_loss_grad(k, v, W1, b1, W2, b2, gamma, beta, ln_eps: float = 1e-6):
    """Loss of one token and its gradients (dW1, db1, dW2, db2) for the MLP inner model."""
    k, v, W1, b1, W2, b2, gamma, beta = (
        _arr(x, np.float64) for x in (k, v, W1, b1, W2, b2, gamma, beta))
    d, hid = W1.shape
    gW1 = np.zeros((d, hid))
    gb1 = np.zeros(hid)
    gW2 = np.zeros((hid, d))
    gb2 = np.zeros(d)
    loss = _load().oracle_mlp_loss_grad_f64(d, hid, ln_eps, _ptr(k), _ptr(v), _ptr(W1), _ptr(b1),
                                            _ptr(W2), _ptr(b2), _ptr(gamma), _ptr(beta),
                                            _ptr(gW1), _ptr(gb1), _ptr(gW2), _ptr(gb2))
    return loss, gW1, gb1, gW2, gb2
