"""ttt_linear_backward_static: the layer backward for callers that cannot
allocate device memory at call time (a host program whose allocator owns all
device memory, or a loop whose latency budget an allocation would break).  Its
workspace is a fixed 32 MiB array inside the library, shared by every call on
a device.

The test calls the entry point through the C ABI (ctypes), with inputs and
outputs the test allocates, and checks it against ttt_linear_backward with a
caller workspace, within the backward tests' tolerance, on two calls in a row
(the second finds the array holding the first call's contents).  It lives in a
file of its own that pytest collects last, and passes alone in a fresh process
as well as after the other tests.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs

pytestmark = pytest.mark.gpu

BAR = 1e-3  # the tolerance of the backward tests (max abs error over the reference's RMS)
KEYS = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")


@pytest.fixture(scope="module")
def ttt(cuda_device):
    from test_sequence_layers_ttt_b200 import _binding
    return _binding


def _p(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def static_call(ttt, w, g, dZ, dW, db, mb):
    B, H, T, d = w.B, w.H, w.T, w.d
    f32 = dict(dtype=torch.float32, device="cuda")
    outs = [torch.empty((B, H, T, d), **f32) for _ in range(3)] + [
        torch.empty((B, H, T), **f32), torch.empty((B, H, d, d), **f32), torch.empty((B, H, d), **f32),
        torch.empty((H, d), **f32), torch.empty((H, d), **f32)]
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = ttt.lib.ttt_linear_backward_static(B, H, T, d, mb, ttt._dtype_code(g["Q"]), 0, w.ln_eps,
                                            *(_p(g[k]) for k in KEYS), _p(dZ), _p(dW), _p(db),
                                            *(_p(o) for o in outs), stream)
    return st, outs


def test_static_workspace_backward_matches_the_workspace_entry_point(ttt):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=3, T=200)
    assert ttt.linear_backward_workspace_size(w.B, w.H, w.T, w.d, 16) <= ttt.STATIC_WORKSPACE_BYTES
    for call, seed in enumerate((5, 6)):  # two calls in a row, different inputs
        g = {k: v.cuda() for k, v in make_inputs(w, seed).items()}
        gen = torch.Generator().manual_seed(seed)
        dZ = torch.randn((w.B, w.H, w.T, w.d), generator=gen).cuda()
        dW = torch.randn((w.B, w.H, w.d, w.d), generator=gen).cuda()
        db = torch.randn((w.B, w.H, w.d), generator=gen).cuda()
        st, got = static_call(ttt, w, g, dZ, dW, db, 16)
        assert st == 0, ttt.status_string(st)
        ref = ttt.ttt_linear_backward(*(g[k] for k in KEYS), dZ, dW, db, mini_batch=16, ln_eps=w.ln_eps)
        torch.cuda.synchronize()
        for name, a, r in zip(("dQ", "dK", "dV", "deta", "dW0", "db0", "dgamma", "dbeta"), got, ref):
            a, r = a.cpu().numpy().astype(np.float64), r.cpu().numpy().astype(np.float64)
            denom = float(np.sqrt(np.mean(r ** 2)))
            err = float(np.abs(a - r).max()) / denom
            assert err <= BAR, f"call {call}, {name}: {err:.2e} of RMS"


def test_static_workspace_refuses_shapes_beyond_its_size(ttt):
    """A shape whose workspace exceeds the fixed array returns TTT_ERR_WORKSPACE
    before anything runs (the pointers are never dereferenced)."""
    B, H, T, d = 8, 12, 2048, 64  # the 125M-layer shape: about 200 MB of states
    assert ttt.linear_backward_workspace_size(B, H, T, d, 16) > ttt.STATIC_WORKSPACE_BYTES
    fake = [ctypes.c_void_p((1 << 40) + i * (1 << 34)) for i in range(19)]
    st = ttt.lib.ttt_linear_backward_static(B, H, T, d, 16, 0, 0, 1e-6, *fake, None)
    assert st == ttt.STATUS.index("TTT_ERR_WORKSPACE")
