"""Pins of the prologue oracle (oracle/prologue.py), CPU only: properties
that any rotary embedding and sigmoid-gated learning rate must have, and the
prologue composed with the scan oracle in Theorem 1's setting."""
from __future__ import annotations

import numpy as np
import pytest

import oracle
from oracle import prologue as op


def weights(seed, D=12, H=3, d=8):
    r = np.random.default_rng(seed)
    tq, tk, tv = (r.normal(0, 1 / np.sqrt(D), (H, D, d)) for _ in range(3))
    tl = r.normal(0, 1, (H, D))
    bl = r.normal(0, 1, (H,))
    return tq, tk, tv, tl, bl


def test_rope_at_position_zero_is_the_identity():
    x = np.random.default_rng(0).normal(size=(2, 1, 1, 8))
    np.testing.assert_array_equal(op.rope(x), x)


def test_rope_preserves_norms_and_pairs():
    x = np.random.default_rng(1).normal(size=(2, 3, 40, 16))
    y = op.rope(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=-1), np.linalg.norm(x, axis=-1), rtol=1e-13)
    # each (i, i + d/2) pair keeps its own norm (a plane rotation per pair)
    d = 16
    nx = x[..., : d // 2] ** 2 + x[..., d // 2:] ** 2
    ny = y[..., : d // 2] ** 2 + y[..., d // 2:] ** 2
    np.testing.assert_allclose(ny, nx, rtol=1e-12)


def test_rope_scores_depend_only_on_the_position_difference():
    r = np.random.default_rng(2)
    q, k = r.normal(size=8), r.normal(size=8)
    T = 30
    Qr = op.rope(np.tile(q, (T, 1)))
    Kr = op.rope(np.tile(k, (T, 1)))
    S = Qr @ Kr.T           # S[m, n] = <R_m q, R_n k>
    for delta in range(-5, 6):
        diag = np.diagonal(S, offset=-delta)
        np.testing.assert_allclose(diag, diag[0], rtol=1e-11, atol=1e-12)


def test_rope_offset_continues_the_sequence():
    x = np.random.default_rng(3).normal(size=(1, 1, 20, 8))
    whole = op.rope(x)
    np.testing.assert_allclose(op.rope(x[..., 12:, :], pos0=12), whole[..., 12:, :], rtol=1e-13)


def test_eta_is_a_sigmoid_gate_over_d():
    tq, tk, tv, tl, bl = weights(4)
    x = np.random.default_rng(5).normal(0, 3, (2, 50, 12))
    _, _, _, eta = op.project(x, tq, tk, tv, tl, bl)
    assert eta.shape == (2, 3, 50)
    assert np.all(eta > 0) and np.all(eta < 1 / 8)
    # a zero logit gives exactly half the base rate
    _, _, _, e0 = op.project(np.zeros((1, 4, 12)), tq, tk, tv, tl, np.zeros(3), eta_base=0.6)
    np.testing.assert_array_equal(e0, np.full((1, 3, 4), 0.6 * 0.5 / 8))


def test_projection_of_a_basis_input_selects_rows():
    tq, tk, tv, tl, bl = weights(6)
    x = np.zeros((1, 1, 12))
    x[0, 0, 5] = 1.0
    Q, K, V, _ = op.project(x, tq, tk, tv, tl, bl, rotary=False)
    np.testing.assert_array_equal(Q[0, :, 0], tq[:, 5, :])
    np.testing.assert_array_equal(K[0, :, 0], tk[:, 5, :])
    np.testing.assert_array_equal(V[0, :, 0], tv[:, 5, :])


def test_prologue_then_scan_is_relative_linear_attention():
    """Theorem 1 through the prologue: plain f, W0 = 0, eta = 1/2, one
    mini-batch, rotary Q and K: z_t = sum_{s<=t} (R_t q_t . R_s k_s) v_s, whose
    scores depend on t - s only through the rotation."""
    tq, tk, tv, tl, bl = weights(7, H=2)
    T = 24
    x = np.random.default_rng(8).normal(0, 1, (1, T, 12))
    Q, K, V, _ = op.project(x, tq, tk, tv, tl, bl)
    eta = np.full((1, 2, T), 0.5)
    Z, _, _ = oracle.ttt_linear(Q, K, V, eta, np.zeros((1, 2, 8, 8)), None, None, None, T,
                                oracle.MODE_PLAIN)
    for h in range(2):
        S = np.tril(Q[0, h] @ K[0, h].T)
        np.testing.assert_allclose(Z[0, h], S @ V[0, h], rtol=1e-11, atol=1e-12)
