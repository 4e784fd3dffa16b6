"""The layer's prologue kernel (projections, learning-rate gate, rotary
embedding; one tcgen05 GEMM with a fused epilogue) against the float64
prologue oracle (oracle/prologue.py), through the C ABI.

Both sides read the same bf16 x and weights.  The kernel accumulates in fp32
and rounds Q, K, V to bf16 (round to nearest): each element may differ from
the float64 value by half a bf16 unit of the value plus the fp32 summation
error, so the bar is 2^-8 of |value| plus 1e-5 of the tensor's RMS.  eta is
fp32: 1e-5 relative.  ("Learning to (Learn at Test Time)", literature record,
Key takeaways bullets 1 and 2.)"""
from __future__ import annotations

import numpy as np
import pytest
import torch

from oracle import prologue as op

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def ttt(cuda_device):
    from test_sequence_layers_ttt_b200 import _binding
    return _binding


def make(B, T, H, dm, seed, d=64):
    g = torch.Generator().manual_seed(seed)
    bf = lambda *shape, std: (torch.randn(shape, generator=g) * std).to(torch.bfloat16)
    x = bf(B, T, dm, std=1.0)
    tq, tk, tv = (bf(H, dm, d, std=dm ** -0.5) for _ in range(3))
    tl = bf(H, dm, std=dm ** -0.5)
    bl = torch.randn(H, generator=g)
    return x, tq, tk, tv, tl, bl


def check(ttt, B, T, H, dm, seed, pos0=0, rotary=True, eta_base=1.0):
    x, tq, tk, tv, tl, bl = make(B, T, H, dm, seed)
    out = ttt.ttt_prologue_forward(x.cuda(), tq.cuda(), tk.cuda(), tv.cuda(), tl.cuda(), bl.cuda(), pos0=pos0,
                                   rotary=rotary, eta_base=eta_base)
    torch.cuda.synchronize()
    ref = op.project(x.float(), tq.float(), tk.float(), tv.float(), tl.float(), bl, eta_base=eta_base,
                     rotary=rotary, pos0=pos0)
    compare(out, ref)


def compare(out, ref, where=""):
    for name, a, r in zip(("Q", "K", "V"), out[:3], ref[:3]):
        a = a.float().cpu().numpy().astype(np.float64)
        rms = float(np.sqrt(np.mean(r ** 2)))
        err = np.abs(a - r) - (2.0 ** -8) * np.abs(r) - 1e-5 * rms
        assert err.max() <= 0, f"{name}{where}: worst excess {err.max():.3e} (rms {rms:.3e})"
    e = out[3].cpu().numpy().astype(np.float64)
    rel = float(np.abs(e - ref[3]).max() / np.abs(ref[3]).max())
    assert rel <= 1e-5, f"eta{where}: {rel:.2e}"


@pytest.mark.parametrize("B,T,H,dm,pos0", [
    (1, 128, 4, 64, 0),       # one row tile, one column tile per projection, K = one stage
    (2, 100, 4, 128, 0),      # rows not a multiple of 128 (the last tile is partial)
    (1, 300, 8, 256, 37),     # several tiles and stages, a position offset
    (2, 256, 12, 768, 0),     # the 125M-layer width (H = 12, d_model = 768)
])
def test_prologue_vs_oracle(ttt, B, T, H, dm, pos0):
    check(ttt, B, T, H, dm, 0, pos0)


def test_prologue_without_rotary_and_scaled_eta(ttt):
    check(ttt, 1, 130, 4, 128, 1, rotary=False, eta_base=0.5)


def test_prologue_long_positions(ttt):
    """Positions near 32k: the rotation angles reach about 3e4 radians."""
    check(ttt, 1, 256, 4, 64, 2, pos0=32768 - 256)


def test_prologue_refuses_unsupported_shapes(ttt):
    x, tq, tk, tv, tl, bl = make(1, 16, 6, 64, 0)  # H = 6 is not a multiple of 4
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_prologue_forward(x.cuda(), tq.cuda(), tk.cuda(), tv.cuda(), tl.cuda(), bl.cuda())
    assert ei.value.status == 6


def test_prologue_full_size_sampled_windows(ttt):
    """The 1.3B layer at 32k tokens in one launch (B = 2, T = 32768, d_model
    2048, H = 32: about 1.1 GB in and out).  Windows of 64 tokens in both
    sequences are checked against the oracle run on each window alone at its
    absolute position: the first window of the second sequence starts at GEMM
    row 32768, where positions restart at 0."""
    B, T, H, dm, W = 2, 32768, 32, 2048, 64
    x, tq, tk, tv, tl, bl = make(B, T, H, dm, 5)
    out = ttt.ttt_prologue_forward(x.cuda(), tq.cuda(), tk.cuda(), tv.cuda(), tl.cuda(), bl.cuda())
    torch.cuda.synchronize()
    weights = (tq.float(), tk.float(), tv.float(), tl.float(), bl)
    for b in range(B):
        for t0 in (0, 8128, 16384 - W // 2, T - W):
            ref = op.project(x[b:b + 1, t0:t0 + W].float(), *weights, pos0=t0)
            got = [o[b:b + 1, :, t0:t0 + W] for o in out]
            compare(got, ref, f" (sequence {b}, tokens {t0}..{t0 + W - 1})")
