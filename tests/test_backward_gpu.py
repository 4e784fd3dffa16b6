"""The TTT-Linear layer backward on the GPU (through the C ABI) against the
float64 backward oracle (oracle/backward.py: torch autograd over a
token-by-token restatement of the scan, pinned to the C oracle and to finite
differences).  Both sides read identical input bits.

Bar: every gradient within 1e-3 of its own RMS (max abs error).  The kernel
runs in fp32; its error grows through the reverse sweep over the mini-batches
and through the second-order LayerNorm terms, so the bar is looser than the
forward's fp32 1e-4.  ("Learning to (Learn at Test Time)", literature record,
Key takeaways bullet 2: the outer loop trains theta_K, theta_V, theta_Q, the
initial weights and the learning rate.)
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import backward as ob
from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

BAR = 1e-3
NAMES = ("dQ", "dK", "dV", "deta", "dW0", "db0", "dgamma", "dbeta")


@pytest.fixture(scope="module")
def ttt(cuda_device):
    from test_sequence_layers_ttt_b200 import _binding
    return _binding


def rms(x):
    return float(np.sqrt(np.mean(np.square(np.asarray(x, dtype=np.float64)))))


def upstream(w, seed, with_state=True):
    g = torch.Generator().manual_seed(1000 + seed)
    dZ = torch.randn((w.B, w.H, w.T, w.d), generator=g)
    dW = torch.randn((w.B, w.H, w.d, w.d), generator=g) if with_state else None
    db = torch.randn((w.B, w.H, w.d), generator=g) if with_state else None
    return dZ, dW, db


def check(ttt, w, inp, dZ, dW, db, mb):
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    cu = lambda t: None if t is None else t.cuda()
    got = ttt.ttt_linear_backward(*(cu(inp[k]) for k in keys), cu(dZ), cu(dW), cu(db), mini_batch=mb,
                                  ln_eps=w.ln_eps)
    torch.cuda.synchronize()
    ref = ob.ttt_linear_backward(*(inp[k] for k in keys), dZ, mb, ln_eps=w.ln_eps,
                                 dW_T=None if dW is None else dW, db_T=None if db is None else db)
    worst = {}
    for name, a, r in zip(NAMES, got, ref):
        a = a.cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), f"{name}: non-finite"
        err = float(np.abs(a - r).max()) / rms(r)
        worst[name] = err
        assert err <= BAR, f"{name}: max err {err:.2e} of RMS > {BAR}"
    return worst


@pytest.mark.parametrize("seed", [0, 1])
@pytest.mark.parametrize("name,shape,mb", [
    ("linear_125m_2k", dict(B=1, H=2, T=48), 16),        # bf16, three mini-batches
    ("linear_125m_2k", dict(B=2, H=3, T=40), 16),        # ragged last mini-batch
    ("linear_125m_2k", dict(B=1, H=2, T=24), 8),
    ("linear_125m_2k", dict(B=1, H=2, T=7), 1),           # online GD
    ("linear_tiny_f32", {}, 16),                          # fp32, d = 16
    ("linear_tiny_f32", dict(d=32, T=40), 4),
])
def test_linear_backward_vs_oracle(ttt, seed, name, shape, mb):
    w = WORKLOADS[name].with_shape(**shape) if shape else WORKLOADS[name]
    inp = make_inputs(w, seed)
    check(ttt, w, inp, *upstream(w, seed), mb)


def test_linear_backward_without_state_gradients(ttt):
    """dW_T, db_T NULL: only the output's gradient flows back."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=64)
    inp = make_inputs(w, 3)
    check(ttt, w, inp, *upstream(w, 3, with_state=False), 16)


def test_linear_backward_125m_heads(ttt):
    """Every head of the 125M-layer shape (B = 8, H = 12, d = 64, b = 16, bf16
    Q/K/V), on 256 tokens (the oracle's autograd loop bounds T)."""
    w = WORKLOADS["linear_125m_2k"].with_shape(T=256)
    inp = make_inputs(w, 0)
    check(ttt, w, inp, *upstream(w, 0), 16)


# Long sequences: the gradients of the first tokens are carried back through every
# later mini-batch, and fp32 rounding grows along that path.  The same steps as the
# oracle, evaluated in float32 on the CPU, miss the float64 result by about 1.5e-2 of
# RMS (dK) at 4096 tokens of the 1.3B-layer shape, so the 1e-3 bar cannot hold for any
# fp32 implementation there.  The bar is four times that fp32 floor, per gradient, and
# never below 1e-3.
FLOOR_FACTOR = 4.0


def check_against_float32_floor(ttt, w, seed):
    """Past 16 mini-batches the bar is FLOOR_FACTOR times the error of the
    oracle's own steps evaluated in float32, and never below BAR."""
    inp = make_inputs(w, seed)
    dZ, dW, db = upstream(w, seed)
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    got = ttt.ttt_linear_backward(*(inp[k].cuda() for k in keys), dZ.cuda(), dW.cuda(), db.cuda(), mini_batch=16,
                                  ln_eps=w.ln_eps)
    torch.cuda.synchronize()
    ref = ob.ttt_linear_backward(*(inp[k] for k in keys), dZ, 16, ln_eps=w.ln_eps, dW_T=dW, db_T=db)
    f32 = ob.ttt_linear_backward(*(inp[k] for k in keys), dZ, 16, ln_eps=w.ln_eps, dW_T=dW, db_T=db,
                                 dtype=torch.float32)
    for name, a, r, f in zip(NAMES, got, ref, f32):
        a = a.cpu().numpy().astype(np.float64)
        assert np.isfinite(a).all(), f"{name}: non-finite"
        floor = float(np.abs(np.asarray(f, dtype=np.float64) - r).max()) / rms(r)
        err = float(np.abs(a - r).max()) / rms(r)
        bar = max(BAR, FLOOR_FACTOR * floor)
        assert err <= bar, f"{name}: max err {err:.2e} of RMS > {bar:.2e} (fp32 floor {floor:.2e})"


def test_linear_backward_long_sequence(ttt):
    """One head of the 1.3B-layer shape over 4096 tokens (256 mini-batches)."""
    check_against_float32_floor(ttt, WORKLOADS["linear_1p3b_32k"].with_shape(B=1, H=1, T=4096), 2)


@pytest.mark.parametrize("T", [1008, 1000])
def test_linear_backward_odd_and_ragged_mini_batch_counts(ttt, T):
    """Three heads of the 1.3B-layer shape.  T = 1008 is 63 whole mini-batches,
    an odd count and a multiple of none of the tensor-core checkpoint pass's
    ring depths (4 and 8), so its rings end part-way through a cycle.  T = 1000
    ends in a ragged mini-batch of 8 tokens: the checkpoints come from the fp32
    pass, and the reverse sweep starts on a short block."""
    check_against_float32_floor(ttt, WORKLOADS["linear_1p3b_32k"].with_shape(B=1, H=3, T=T), 3)


@pytest.fixture(scope="module")
def full_size_run(ttt):
    """The whole 1.3B-layer workload at 32k tokens (B = 2, H = 32: the bench's launch), run once."""
    w = WORKLOADS["linear_1p3b_32k"]
    inp = make_inputs(w, 0)
    dZ, dW, db = upstream(w, 0)
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    got = ttt.ttt_linear_backward(*(inp[k].cuda() for k in keys), dZ.cuda(), dW.cuda(), db.cuda(), mini_batch=16,
                                  ln_eps=w.ln_eps)
    torch.cuda.synchronize()
    return w, inp, (dZ, dW, db), [g.cpu() for g in got[:6]]


@pytest.mark.parametrize("scan", [(0, 5), (1, 27)])
def test_linear_backward_full_size_sampled_scans(full_size_run, scan):
    """The per-scan gradients (dQ, dK, dV, deta, dW0, db0) of one sampled (batch, head) scan of
    the full-size run, checked against the oracle run on that scan alone (the scans are
    independent; dgamma, dbeta, sums over the batch, are left to the smaller cases).  Bar:
    four times the fp32 floor of that scan, never below 1e-3."""
    w, inp, (dZ, dW, db), got = full_size_run
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    b, h = scan
    one = {k: inp[k][b:b + 1, h:h + 1] for k in ("Q", "K", "V", "eta", "W0", "b0")}
    one.update({k: inp[k][h:h + 1] for k in ("gamma", "beta")})
    sl = lambda t: t[b:b + 1, h:h + 1]
    args = [one[k] for k in keys]
    ref = ob.ttt_linear_backward(*args, sl(dZ), 16, ln_eps=w.ln_eps, dW_T=sl(dW), db_T=sl(db))
    f32 = ob.ttt_linear_backward(*args, sl(dZ), 16, ln_eps=w.ln_eps, dW_T=sl(dW), db_T=sl(db), dtype=torch.float32)
    for name, a, r, f in zip(NAMES[:6], got, ref, f32):
        a = sl(a).numpy().astype(np.float64)
        assert np.isfinite(a).all(), f"{name}: non-finite"
        floor = float(np.abs(np.asarray(f, dtype=np.float64) - r).max()) / rms(r)
        err = float(np.abs(a - r).max()) / rms(r)
        bar = max(BAR, FLOOR_FACTOR * floor)
        assert err <= bar, f"{name}: max err {err:.2e} of RMS > {bar:.2e} (fp32 floor {floor:.2e})"


def test_linear_backward_empty_sequence(ttt):
    """T = 0: dW0 = dW_T, db0 = db_T, dgamma = dbeta = 0."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=0)
    g = {k: v.cuda() for k, v in make_inputs(w, 1).items()}
    dZ, dW, db = (None if t is None else t.cuda() for t in upstream(w, 1))
    out = ttt.ttt_linear_backward(g["Q"], g["K"], g["V"], g["eta"], g["W0"], g["b0"], g["gamma"], g["beta"], dZ,
                                  dW, db)
    torch.cuda.synchronize()
    assert torch.equal(out[4], dW) and torch.equal(out[5], db)
    assert not out[6].any() and not out[7].any()


def test_linear_backward_refuses_small_workspace_and_plain_mode(ttt):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=1, T=32)
    g = {k: v.cuda() for k, v in make_inputs(w, 0).items()}
    dZ = torch.zeros((1, 1, 32, 64), device="cuda")
    args = (g["Q"], g["K"], g["V"], g["eta"], g["W0"], g["b0"], g["gamma"], g["beta"], dZ)
    need = ttt.linear_backward_workspace_size(1, 1, 32, 64, 16)
    small = torch.empty(need - 16, dtype=torch.uint8, device="cuda")
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_linear_backward(*args, workspace=small)
    assert ei.value.status == 9
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_linear_backward(*args, mode="plain")
    assert ei.value.status == 6


def test_linear_backward_is_deterministic(ttt):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=3, H=2, T=64)
    g = {k: v.cuda() for k, v in make_inputs(w, 4).items()}
    dZ, dW, db = (t.cuda() for t in upstream(w, 4))
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    a = ttt.ttt_linear_backward(*(g[k] for k in keys), dZ, dW, db)
    b = ttt.ttt_linear_backward(*(g[k] for k in keys), dZ, dW, db)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))
