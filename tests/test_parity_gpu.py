"""Parity of the CUDA library (through the C ABI) against the float64 oracle.

Bar (stated for the TTT forward scan): max |GPU - oracle| <= 1e-4 * RMS(Z)
with fp32 Q/K/V and <= 3e-3 * RMS(Z) with bf16 Q/K/V and fp32 state.  The
final state is held to the same factor times its own RMS.  Both sides consume
identical input bits from the seeded generators.
"""
from __future__ import annotations

import numpy as np
import pytest
import torch

import oracle
from test_sequence_layers_ttt_b200.inputs import (MODE_PLAIN, WORKLOADS, make_inputs,
                                                  select_heads)

pytestmark = pytest.mark.gpu

TOL = {"f32": 1e-4, "bf16": 3e-3}
LINEAR_KEYS = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
MLP_KEYS = ("Q", "K", "V", "eta", "W1_0", "b1_0", "W2_0", "b2_0", "gamma", "beta")


@pytest.fixture(scope="module")
def ttt(cuda_device):
    from test_sequence_layers_ttt_b200 import _binding
    return _binding


def to_cuda(inp):
    return {k: (None if v is None else v.cuda()) for k, v in inp.items()}


def rms(x):
    return float(np.sqrt(np.mean(np.square(x, dtype=np.float64))))


def assert_close(got, ref, factor, what, denom=None):
    got = np.asarray(got, dtype=np.float64)
    d = rms(ref) if denom is None else denom
    err = float(np.abs(got - ref).max()) if got.size else 0.0
    assert np.isfinite(got).all(), f"{what}: non-finite values"
    assert err <= factor * d, f"{what}: max err {err:.3e} > {factor:g} * RMS {d:.3e}"
    return err / d if d else 0.0


def gpu_linear(ttt, w, inp, impl="auto", mini_batch=None):
    g = to_cuda(inp)
    plain = w.mode == MODE_PLAIN
    Z, W_T, b_T = ttt.ttt_linear_forward(
        g["Q"], g["K"], g["V"], g["eta"], g["W0"], None if plain else g["b0"],
        None if plain else g["gamma"], None if plain else g["beta"],
        mini_batch=mini_batch or w.mini_batch, mode="plain" if plain else "ln",
        ln_eps=w.ln_eps, impl=impl)
    torch.cuda.synchronize()
    return Z.cpu().numpy(), W_T.cpu().numpy(), None if b_T is None else b_T.cpu().numpy()


def oracle_linear(w, inp, mini_batch=None):
    return oracle.ttt_linear(*(inp[k] for k in LINEAR_KEYS), mini_batch or w.mini_batch, w.mode,
                             w.ln_eps)


def compare_linear(ttt, w, inp, impl="auto", mini_batch=None):
    Z, W_T, b_T = gpu_linear(ttt, w, inp, impl, mini_batch)
    Zo, Wo, bo = oracle_linear(w, inp, mini_batch)
    f = TOL[w.dtype]
    e = assert_close(Z, Zo, f, "Z")
    assert_close(W_T, Wo, f, "W_T")
    if b_T is not None and np.any(bo):
        assert_close(b_T, bo, f, "b_T")
    return e


# ---------------------------------------------------------------- TTT-Linear

@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("impl", ["auto", "generic"])
def test_linear_tiny_f32(ttt, seed, impl):
    w = WORKLOADS["linear_tiny_f32"]
    compare_linear(ttt, w, make_inputs(w, seed), impl)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_theorem1_f32(ttt, seed):
    """Theorem-1 workload, full size: also equals causal linear attention."""
    w = WORKLOADS["theorem1_f32"]
    inp = make_inputs(w, seed)
    compare_linear(ttt, w, inp)
    Z, _, _ = gpu_linear(ttt, w, inp)
    Q, K, V = (inp[k].double() for k in "QKV")
    Zref = (torch.tril(Q @ K.transpose(-1, -2)) @ V).numpy()
    assert_close(Z, Zref, TOL["f32"], "Z vs linear attention")


@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("name,shape", [
    ("linear_125m_2k", dict(B=2, H=3, T=200)),       # several chunks + ragged tail (200 = 12*16 + 8)
    ("linear_1p3b_32k", dict(B=1, H=4, T=1000)),
])
@pytest.mark.parametrize("impl", ["auto", "generic"])
def test_linear_bf16_reduced(ttt, seed, name, shape, impl):
    w = WORKLOADS[name].with_shape(**shape)
    compare_linear(ttt, w, make_inputs(w, seed), impl)


# the tensor-core families of TTT-Linear: warp-level mma with the state in
# registers, and the state products on tcgen05 with TMEM accumulators
TC_LINEAR = ["tensorcore", "tcgen05"]


@pytest.mark.parametrize("impl", ["auto"] + TC_LINEAR)
def test_linear_125m_full(ttt, impl):
    w = WORKLOADS["linear_125m_2k"]
    compare_linear(ttt, w, make_inputs(w, 0), impl)


@pytest.mark.parametrize("impl", TC_LINEAR)
@pytest.mark.parametrize("seed", [0, 1, 2])
@pytest.mark.parametrize("shape", [dict(B=1, H=1, T=16), dict(B=1, H=1, T=32), dict(B=1, H=2, T=48),
                                   dict(B=2, H=3, T=256), dict(B=1, H=4, T=1024)])
def test_linear_tensorcore_shapes(ttt, seed, shape, impl):
    """The tensor-core families on 1, 2, 3, 16 and 64 chunks (every ring wraps)."""
    w = WORKLOADS["linear_1p3b_32k"].with_shape(**shape)
    compare_linear(ttt, w, make_inputs(w, seed), impl)


@pytest.mark.parametrize("impl", TC_LINEAR)
def test_linear_tensorcore_matches_generic_closely(ttt, impl):
    """The CUDA families agree far inside the oracle tolerance."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=2, T=512)
    inp = make_inputs(w, 9)
    Zt, Wt_, _ = gpu_linear(ttt, w, inp, impl)
    Zg, Wg, _ = gpu_linear(ttt, w, inp, "generic")
    assert_close(Zt, Zg, 1e-3, f"Z {impl} vs generic")
    assert_close(Wt_, Wg, 1e-3, f"W_T {impl} vs generic")


@pytest.mark.parametrize("impl", TC_LINEAR + ["generic"])
@pytest.mark.parametrize("offset", [4.0, -2.5])
def test_linear_bias_with_large_mean(ttt, impl, offset):
    """b0 with a mean far above the spread of x W (b0 = offset + N(0, 0.02^2)):
    the mean of y = x W + b is then large against its spread, where a one-pass
    variance in fp32 would cancel; W0 gets a row-mean offset as well."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=2, T=512)
    inp = make_inputs(w, 11)
    gen = torch.Generator().manual_seed(123)
    inp["b0"] = (offset + 0.02 * torch.randn(inp["b0"].shape, generator=gen)).float()
    inp["W0"] = (inp["W0"] + 0.3 * torch.randn(inp["W0"].shape[:-1] + (1,), generator=gen)).float()
    compare_linear(ttt, w, inp, impl)


_FAULT_CHILD = r"""
import sys, numpy as np, torch
sys.path.insert(0, sys.argv[2])
import oracle
from test_sequence_layers_ttt_b200 import _binding as ttt
from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs
keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
impl = sys.argv[1]
w = WORKLOADS["linear_1p3b_32k"].with_shape(B=1, H=2, T=256)
g = {k: v.cuda() for k, v in make_inputs(w, 0).items()}
try:
    ttt.ttt_linear_forward(*(g[k] for k in keys), impl=impl)
    print("NO_TIMEOUT")
except ttt.TTTError as e:
    print("STATUS", e.status)
torch.cuda.synchronize()
# the same context, a sequence of three chunks (chunk 3 does not exist, so the hook never fires)
w3 = w.with_shape(T=48)
inp = make_inputs(w3, 1)
Z, W_T, b_T = ttt.ttt_linear_forward(*(inp[k].cuda() for k in keys), impl=impl)
torch.cuda.synchronize()
Zo, Wo, bo = oracle.ttt_linear(*(inp[k] for k in keys), 16)
err = float(np.abs(Z.cpu().numpy() - Zo).max()) / float(np.sqrt(np.mean(Zo ** 2)))
print("AFTER", err)
"""


@pytest.mark.parametrize("impl", TC_LINEAR)
def test_linear_bounded_wait_times_out_and_context_survives(ttt, impl, tmp_path):
    """Fault injection on the host side of a bounded wait, in a child process
    (the library reads its environment once per process): the producer is told
    never to load chunk 3, so the consumers' wait for it runs out (about a
    second), the kernel drains its loads and tensor-core work and returns, and
    the call reports TTT_ERR_TIMEOUT.  A later call on the same context is
    correct."""
    import os
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, TTT_CHECK="1", TTT_DEBUG_DROP_CHUNK="3")
    r = subprocess.run([sys.executable, "-c", _FAULT_CHILD, impl, root], env=env, capture_output=True,
                       text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = r.stdout.split("\n")
    assert "STATUS 8" in lines, r.stdout
    after = [float(l.split()[1]) for l in lines if l.startswith("AFTER")]
    assert after and after[0] <= TOL["bf16"], r.stdout


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_linear_1p3b_32k_full_all_scans(ttt, seed):
    """The benchmarked launch: all 64 scans of 32k tokens on the GPU, every one
    checked end to end against the oracle."""
    w = WORKLOADS["linear_1p3b_32k"]
    inp = make_inputs(w, seed)
    Z, W_T, b_T = gpu_linear(ttt, w, inp)
    Zo, Wo, bo = oracle_linear(w, inp)
    f = TOL["bf16"]
    assert_close(Z, Zo, f, "Z")
    assert_close(W_T, Wo, f, "W_T")
    assert_close(b_T, bo, f, "b_T")


@pytest.mark.parametrize("impl", TC_LINEAR)
def test_linear_1p3b_32k_full_each_tensorcore_family(ttt, impl):
    """Each tensor-core family on the full 1.3B/32k launch, all 64 scans."""
    w = WORKLOADS["linear_1p3b_32k"]
    compare_linear(ttt, w, make_inputs(w, 1), impl)


@pytest.mark.parametrize("mb", [1, 2, 4, 8, 32, 64])
def test_linear_mini_batch_sizes(ttt, mb):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=192)
    compare_linear(ttt, w, make_inputs(w, 3), mini_batch=mb)


@pytest.mark.parametrize("d", [16, 32, 64])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("mode", [0, 1])
def test_linear_dims_dtypes_modes(ttt, d, dtype, mode):
    w = WORKLOADS["linear_tiny_f32"].with_shape(B=2, H=2, T=72, d=d, dtype=dtype, mode=mode)
    compare_linear(ttt, w, make_inputs(w, 4))


@pytest.mark.parametrize("T", [0, 1, 15, 17])
def test_linear_short_and_empty_sequences(ttt, T):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=T)
    inp = make_inputs(w, 5)
    Z, W_T, b_T = gpu_linear(ttt, w, inp)
    if T == 0:
        np.testing.assert_array_equal(W_T, inp["W0"].numpy())
        np.testing.assert_array_equal(b_T, inp["b0"].numpy())
        assert Z.size == 0
    else:
        compare_linear(ttt, w, inp)


@pytest.mark.parametrize("impl", ["generic"] + TC_LINEAR)
def test_linear_in_place_state_and_continuation(ttt, impl):
    """W_T may be W0 (in-place).  Splitting the sequence at a mini-batch
    boundary and feeding the state back continues the same computation:
    bit for bit in the generic family, up to rounding in the tensor-core one."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=2, T=256)
    g = to_cuda(make_inputs(w, 6))
    args = lambda sl: [g[k][:, :, sl].contiguous() for k in ("Q", "K", "V", "eta")]
    Zf, Wf, bf = ttt.ttt_linear_forward(*args(slice(None)), g["W0"], g["b0"], g["gamma"], g["beta"],
                                        impl=impl)
    W, b = g["W0"].clone(), g["b0"].clone()
    Za, _, _ = ttt.ttt_linear_forward(*args(slice(0, 128)), W, b, g["gamma"], g["beta"], W_T=W, b_T=b,
                                      impl=impl)
    Zb, _, _ = ttt.ttt_linear_forward(*args(slice(128, None)), W, b, g["gamma"], g["beta"], W_T=W,
                                      b_T=b, impl=impl)
    torch.cuda.synchronize()
    if impl == "generic":
        assert torch.equal(torch.cat([Za, Zb], dim=2), Zf)
        assert torch.equal(W, Wf) and torch.equal(b, bf)
    else:
        # the tensor-core family reaches the first chunk after the split by a
        # different (algebraically equal) path, so only rounding may differ
        assert_close(torch.cat([Za, Zb], dim=2).cpu().numpy(), Zf.cpu().numpy(), 1e-4, "Z continuation")
        assert_close(W.cpu().numpy(), Wf.cpu().numpy(), 1e-4, "W continuation")


@pytest.mark.parametrize("impl", ["auto", "generic"] + TC_LINEAR)
def test_linear_deterministic(ttt, impl):
    w = WORKLOADS["linear_1p3b_32k"].with_shape(B=2, H=4, T=512)
    g = to_cuda(make_inputs(w, 7))
    a = ttt.ttt_linear_forward(*(g[k] for k in LINEAR_KEYS), impl=impl)
    b = ttt.ttt_linear_forward(*(g[k] for k in LINEAR_KEYS), impl=impl)
    torch.cuda.synchronize()
    assert all(torch.equal(x, y) for x, y in zip(a, b))


@pytest.mark.parametrize("impl", TC_LINEAR)
def test_linear_tensorcore_refuses_other_shapes(ttt, impl):
    w = WORKLOADS["linear_tiny_f32"]
    g = to_cuda(make_inputs(w, 0))
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_linear_forward(*(g[k] for k in LINEAR_KEYS), impl=impl)
    assert ei.value.status == 6


def test_linear_host_buffers_end_to_end(ttt):
    """CPU tensors in, CPU tensors out: the same numbers as the device path."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=3, T=96)
    inp = make_inputs(w, 8)
    Zh, Wh, bh = ttt.ttt_linear_forward(*(inp[k] for k in LINEAR_KEYS))
    assert Zh.device.type == "cpu"
    Zd, Wd, bd = gpu_linear(ttt, w, inp)
    np.testing.assert_array_equal(Zh.numpy(), Zd)
    np.testing.assert_array_equal(Wh.numpy(), Wd)


def test_linear_host_buffers_on_an_explicit_stream(ttt):
    """CPU tensors with a caller stream: the copies in, the scan and the copies
    back are all ordered on that stream, so the results equal the device call
    even while other work is queued on the default stream."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=3, T=256)
    inp = make_inputs(w, 9)
    side = torch.cuda.Stream()
    busy = torch.randn(4096, 4096, device="cuda")
    for _ in range(8):
        busy = busy @ busy  # keep the default stream occupied
        busy /= busy.norm()
    Zh, Wh, bh = ttt.ttt_linear_forward(*(inp[k] for k in LINEAR_KEYS), stream=side)
    torch.cuda.synchronize()
    Zd, Wd, bd = gpu_linear(ttt, w, inp)
    np.testing.assert_array_equal(Zh.numpy(), Zd)
    np.testing.assert_array_equal(Wh.numpy(), Wd)
    np.testing.assert_array_equal(bh.numpy(), bd)


@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_linear_host_pipeline_uneven_groups(ttt, mode):
    """The host path cuts the scans into groups on several streams; groups of
    unequal size, both modes, and the result equals the device call bit for bit."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=5, T=64)
    if mode == "plain":
        w = w.with_shape(mode=MODE_PLAIN)
    inp = make_inputs(w, 3)
    plain = mode == "plain"
    host = ttt.ttt_linear_forward(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"],
                                  None if plain else inp["b0"], None if plain else inp["gamma"],
                                  None if plain else inp["beta"], mode=mode)
    dev = gpu_linear(ttt, w, inp)
    np.testing.assert_array_equal(host[0].numpy(), dev[0])
    np.testing.assert_array_equal(host[1].numpy(), dev[1])
    if not plain:
        np.testing.assert_array_equal(host[2].numpy(), dev[2])


# ------------------------------------------------------------------ TTT-Linear decode

def gpu_decode_pieces(ttt, w, inp, cuts, mini_batch=None):
    """Decode calls over [0, T) cut at `cuts`, the state carried on the GPU."""
    mb = mini_batch or w.mini_batch
    g = to_cuda(inp)
    plain = w.mode == MODE_PLAIN
    W = g["W0"].clone()
    b = None if plain else g["b0"].clone()
    W_mb = torch.zeros_like(W)
    b_mb = None if plain else torch.zeros_like(b)
    T = g["Q"].shape[2]
    bounds = [0, *cuts, T]
    Zs = []
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = lambda x: x[:, :, a:c].contiguous()
        Zs.append(ttt.ttt_linear_decode(sl(g["Q"]), sl(g["K"]), sl(g["V"]), sl(g["eta"]), W, b, W_mb, b_mb,
                                        None if plain else g["gamma"], None if plain else g["beta"],
                                        pos0=a % mb, mini_batch=mb, mode="plain" if plain else "ln",
                                        ln_eps=w.ln_eps))
    torch.cuda.synchronize()
    out = [torch.cat(Zs, dim=2), W, b, W_mb, b_mb]
    return [None if o is None else o.cpu().numpy() for o in out]


def oracle_decode_pieces(w, inp, cuts, mini_batch=None):
    mb = mini_batch or w.mini_batch
    T = inp["Q"].shape[2]
    W, b, W_mb, b_mb = inp["W0"], inp["b0"], None, None
    bounds = [0, *cuts, T]
    Zs = []
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = lambda x: x[:, :, a:c]
        Z, W, b, W_mb, b_mb = oracle.ttt_linear_decode(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]),
                                                       sl(inp["eta"]), W, b, W_mb, b_mb, inp["gamma"],
                                                       inp["beta"], mb, a % mb, w.mode, w.ln_eps)
        Zs.append(Z)
    return [np.concatenate(Zs, axis=2), W, b, W_mb, b_mb]


def compare_decode(out, ref, f, plain):
    assert_close(out[0], ref[0], f, "Z")
    for name, i in (("W", 1), ("W_mb", 3)):
        assert_close(out[i], ref[i], f, name)
    if not plain:
        for name, i in (("b", 2), ("b_mb", 4)):
            assert_close(out[i], ref[i], f, name)


@pytest.mark.parametrize("name,shape,mb,cuts", [
    ("linear_125m_2k", dict(B=1, H=2, T=96), 16, [5, 6, 21, 40, 64, 79]),
    ("linear_125m_2k", dict(B=2, H=3, T=100), 32, [1, 33, 50]),
    ("linear_tiny_f32", {}, 16, [3, 17, 18, 47]),
    ("linear_tiny_f32", {}, 8, [1, 2, 3, 12, 29]),
    ("theorem1_f32", dict(B=1, H=2, T=80), 80, [7, 30, 31]),
    ("linear_125m_2k", dict(B=1, H=2, T=24), 1, [5, 9]),          # b = 1: online GD
    ("linear_125m_2k", dict(B=1, H=2, T=48, d=32), 16, [5, 21]),  # d = 32: generic family
])
def test_linear_decode_pieces_vs_oracle(ttt, name, shape, mb, cuts):
    """Decode calls cut anywhere (inside mini-batches, ragged tails) against the
    oracle's decode over the same pieces."""
    w = WORKLOADS[name].with_shape(**shape) if shape else WORKLOADS[name]
    inp = make_inputs(w, 2)
    out = gpu_decode_pieces(ttt, w, inp, cuts, mb)
    ref = oracle_decode_pieces(w, inp, cuts, mb)
    compare_decode(out, ref, TOL[w.dtype], w.mode == MODE_PLAIN)


def test_linear_decode_token_by_token_equals_forward_oracle(ttt):
    """Single-token decode steps over a stream reproduce the oracle's forward scan."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=40)
    inp = make_inputs(w, 3)
    out = gpu_decode_pieces(ttt, w, inp, list(range(1, 40)))
    Zo, Wo, bo = oracle_linear(w, inp)
    f = TOL[w.dtype]
    assert_close(out[0], Zo, f, "Z")
    assert_close(out[1], Wo, f, "W")
    assert_close(out[2], bo, f, "b")


def test_linear_decode_full_shape_one_token_per_call(ttt):
    """The decode bench's launch: every (batch, head) stream of the 1.3B-layer
    shape (B = 2, H = 32) decoded one token per call over three mini-batches,
    outputs and both states against the oracle's decode of the same calls."""
    w = WORKLOADS["decode_1p3b"].with_shape(T=48)
    inp = make_inputs(w, 6)
    cuts = list(range(1, 48))
    compare_decode(gpu_decode_pieces(ttt, w, inp, cuts), oracle_decode_pieces(w, inp, cuts), TOL[w.dtype],
                   w.mode == MODE_PLAIN)


def test_linear_decode_one_call_is_the_generic_forward(ttt):
    """From a mini-batch boundary, one decode call at d = 32 (generic family)
    runs the generic forward scan operation for operation."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=2, T=72, d=32)
    inp = make_inputs(w, 4)
    dec = gpu_decode_pieces(ttt, w, inp, [])
    fwd = gpu_linear(ttt, w, inp, impl="generic")
    np.testing.assert_array_equal(dec[0], fwd[0])
    np.testing.assert_array_equal(dec[1], fwd[1])
    np.testing.assert_array_equal(dec[2], fwd[2])
    # 72 = 4 * 16 + 8 tokens: the call ends inside a mini-batch, whose start
    # state is the state after 64 tokens
    first = {k: (v[:, :, :64].contiguous() if k in ("Q", "K", "V", "eta") else v) for k, v in inp.items()}
    fwd64 = gpu_linear(ttt, w.with_shape(T=64), first, impl="generic")
    np.testing.assert_array_equal(dec[3], fwd64[1])
    np.testing.assert_array_equal(dec[4], fwd64[2])


@pytest.mark.parametrize("mode", ["ln", "plain"])
def test_linear_decode_register_kernel_matches_generic_forward(ttt, mode):
    """d = 64 decode (state in registers, token-serial) against the generic
    forward scan: the same fp32 arithmetic in another order."""
    w = WORKLOADS["linear_125m_2k"].with_shape(B=2, H=2, T=72, mode=MODE_PLAIN if mode == "plain" else 0)
    inp = make_inputs(w, 6)
    dec = gpu_decode_pieces(ttt, w, inp, [])
    fwd = gpu_linear(ttt, w, inp, impl="generic")
    assert_close(dec[0], fwd[0].astype(np.float64), 1e-4, "Z")
    assert_close(dec[1], fwd[1].astype(np.float64), 1e-4, "W")
    if mode == "ln":
        assert_close(dec[2], fwd[2].astype(np.float64), 1e-4, "b", denom=max(rms(fwd[2]), rms(fwd[1])))


def test_linear_decode_empty_call_keeps_state(ttt):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=2, T=0)
    g = to_cuda(make_inputs(w, 5))
    W, b = g["W0"].clone(), g["b0"].clone()
    W_mb, b_mb = W + 0.5, b - 0.5
    W_mb0, b_mb0 = W_mb.clone(), b_mb.clone()
    Z = ttt.ttt_linear_decode(g["Q"], g["K"], g["V"], g["eta"], W, b, W_mb, b_mb, g["gamma"], g["beta"],
                              pos0=5, mini_batch=16)
    torch.cuda.synchronize()
    assert Z.shape == (1, 2, 0, 64)
    assert torch.equal(W, g["W0"]) and torch.equal(W_mb, W_mb0) and torch.equal(b_mb, b_mb0)


def test_linear_decode_bad_position(ttt):
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=1, T=4)
    g = to_cuda(make_inputs(w, 0))
    W, b = g["W0"].clone(), g["b0"].clone()
    with pytest.raises(ttt.TTTError) as ei:
        ttt.ttt_linear_decode(g["Q"], g["K"], g["V"], g["eta"], W, b, W.clone(), b.clone(), g["gamma"],
                              g["beta"], pos0=16, mini_batch=16)
    assert ei.value.status == 2


# ------------------------------------------------------------------ TTT-MLP

# the tensor-core families: one CTA per scan, and each scan's hidden units
# split over a 2-CTA cluster
TC_MLP = ["tensorcore", "tensorcore_split"]

def gpu_mlp(ttt, w, inp, mini_batch=None, impl="auto"):
    g = to_cuda(inp)
    out = ttt.ttt_mlp_forward(*(g[k] for k in MLP_KEYS), mini_batch=mini_batch or w.mini_batch,
                              ln_eps=w.ln_eps, impl=impl)
    torch.cuda.synchronize()
    return [o.cpu().numpy() for o in out]


def oracle_mlp(w, inp, mini_batch=None):
    return oracle.ttt_mlp(*(inp[k] for k in MLP_KEYS), mini_batch or w.mini_batch, w.ln_eps)


def compare_mlp(ttt, w, inp, mini_batch=None, pairs=None, impl="auto"):
    out = gpu_mlp(ttt, w, inp, mini_batch, impl)
    if pairs is not None:
        ref = oracle_mlp(w, select_heads(inp, pairs), mini_batch)
        out = [np.stack([o[bb, hh] for bb, hh in pairs])[None] for o in out]
    else:
        ref = oracle_mlp(w, inp, mini_batch)
    f = TOL[w.dtype]
    assert_close(out[0], ref[0], f, "Z")
    for name, o, r in zip(("W1_T", "b1_T", "W2_T", "b2_T"), out[1:], ref[1:]):
        scale = rms(r) if np.any(r) else 1.0
        assert_close(o, r, f, name, denom=max(scale, 1e-3 * rms(ref[1])))


STATE_MLP = ("W1_0", "b1_0", "W2_0", "b2_0")


def gpu_mlp_decode_pieces(ttt, w, inp, cuts, mb, impl="auto"):
    g = to_cuda(inp)
    run = [g[k].clone() for k in STATE_MLP]
    start = [torch.zeros_like(x) for x in run]
    T = g["Q"].shape[2]
    bounds = [0, *cuts, T]
    Zs = []
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = lambda x: x[:, :, a:c].contiguous()
        Zs.append(ttt.ttt_mlp_decode(sl(g["Q"]), sl(g["K"]), sl(g["V"]), sl(g["eta"]), *run, *start, g["gamma"],
                                     g["beta"], pos0=a % mb, mini_batch=mb, ln_eps=w.ln_eps, impl=impl))
    torch.cuda.synchronize()
    return [x.cpu().numpy() for x in (torch.cat(Zs, dim=2), *run, *start)]


def oracle_mlp_decode_pieces(w, inp, cuts, mb):
    T = inp["Q"].shape[2]
    run, start = [inp[k] for k in STATE_MLP], [None] * 4
    bounds = [0, *cuts, T]
    Zs = []
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = lambda x: x[:, :, a:c]
        out = oracle.ttt_mlp_decode(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["eta"]), *run, *start,
                                    inp["gamma"], inp["beta"], mb, a % mb, w.ln_eps)
        Zs.append(out[0])
        run, start = list(out[1:5]), list(out[5:9])
    return [np.concatenate(Zs, axis=2), *run, *start]


@pytest.mark.parametrize("shape,mb,cuts,impl", [
    (dict(B=1, H=2, T=80), 16, [5, 6, 21, 40, 63], "auto"),
    (dict(B=1, H=2, T=72), 32, [1, 33, 50], "auto"),
    (dict(B=1, H=2, T=40), 8, [3, 4, 19], "auto"),
    (dict(B=1, H=2, T=24), 1, [5, 9], "auto"),
    (dict(B=1, H=2, T=48, dtype="f32"), 16, [7, 30], "auto"),
    (dict(B=2, H=3, T=40), 16, [5, 21], "auto"),
    (dict(B=1, H=2, T=80), 16, [5, 6, 21, 40, 63], "generic"),
    (dict(B=1, H=2, T=72), 32, [1, 33, 50], "generic"),
])
def test_mlp_decode_pieces_vs_oracle(ttt, shape, mb, cuts, impl):
    """TTT-MLP decode calls cut anywhere against the oracle's decode over the same
    pieces: outputs, running state and mini-batch start state (the decode kernel,
    and the generic scan run from inside a mini-batch)."""
    w = WORKLOADS["mlp_8k"].with_shape(**shape)
    inp = make_inputs(w, 3)
    out = gpu_mlp_decode_pieces(ttt, w, inp, cuts, mb, impl)
    ref = oracle_mlp_decode_pieces(w, inp, cuts, mb)
    f = TOL[w.dtype]
    assert_close(out[0], ref[0], f, "Z")
    names = ("W1", "b1", "W2", "b2", "W1_mb", "b1_mb", "W2_mb", "b2_mb")
    for name, o, r in zip(names, out[1:], ref[1:]):
        scale = rms(r) if np.any(r) else 1.0
        assert_close(o, r, f, name, denom=max(scale, 1e-3 * rms(ref[1])))


def test_mlp_decode_full_shape_one_token_per_call(ttt):
    """The TTT-MLP decode bench's launch (B = 4, H = 12, hidden 256) decoded one
    token per call over two and a half mini-batches, outputs and both states
    against the oracle's decode of the same calls."""
    w = WORKLOADS["decode_mlp_8k"].with_shape(T=40)
    inp = make_inputs(w, 7)
    cuts = list(range(1, 40))
    out = gpu_mlp_decode_pieces(ttt, w, inp, cuts, w.mini_batch)
    ref = oracle_mlp_decode_pieces(w, inp, cuts, w.mini_batch)
    f = TOL[w.dtype]
    assert_close(out[0], ref[0], f, "Z")
    names = ("W1", "b1", "W2", "b2", "W1_mb", "b1_mb", "W2_mb", "b2_mb")
    for name, o, r in zip(names, out[1:], ref[1:]):
        scale = rms(r) if np.any(r) else 1.0
        assert_close(o, r, f, name, denom=max(scale, 1e-3 * rms(ref[1])))


def test_mlp_decode_token_by_token_equals_forward_oracle(ttt):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=24)
    inp = make_inputs(w, 4)
    out = gpu_mlp_decode_pieces(ttt, w, inp, list(range(1, 24)), 16)
    ref = oracle_mlp(w, inp)
    assert_close(out[0], ref[0], TOL[w.dtype], "Z")


def test_mlp_decode_register_kernel_matches_generic_forward(ttt):
    """The decode kernel (running state in registers, token-serial) against the
    generic forward scan: the same fp32 arithmetic in another order."""
    w = WORKLOADS["mlp_8k"].with_shape(B=2, H=2, T=64)
    inp = make_inputs(w, 6)
    dec = gpu_mlp_decode_pieces(ttt, w, inp, [], 16)
    fwd = gpu_mlp(ttt, w, inp, impl="generic")
    for name, a, b in zip(("Z", "W1", "b1", "W2", "b2"), dec[:5], fwd):
        assert_close(a, b.astype(np.float64), 1e-4, name, denom=max(rms(b), 1e-3))


def test_mlp_decode_empty_call_keeps_state(ttt):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=0)
    g = to_cuda(make_inputs(w, 2))
    run = [g[k].clone() for k in STATE_MLP]
    start = [x + 0.5 for x in run]
    start0 = [x.clone() for x in start]
    Z = ttt.ttt_mlp_decode(g["Q"], g["K"], g["V"], g["eta"], *run, *start, g["gamma"], g["beta"], pos0=5)
    torch.cuda.synchronize()
    assert Z.shape == (1, 2, 0, 64)
    assert all(torch.equal(a, g[k]) for a, k in zip(run, STATE_MLP))
    assert all(torch.equal(a, b) for a, b in zip(start, start0))


def test_mlp_decode_one_call_is_the_generic_forward(ttt):
    """From a mini-batch boundary, one generic decode call runs the generic
    forward scan operation for operation (the start state read from the
    caller's buffer instead of shared memory)."""
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=64)
    inp = make_inputs(w, 5)
    dec = gpu_mlp_decode_pieces(ttt, w, inp, [], 16, impl="generic")
    fwd = gpu_mlp(ttt, w, inp, impl="generic")
    for a, b in zip(dec[:5], fwd):
        np.testing.assert_array_equal(a, b)
    for a, b in zip(dec[5:], fwd[1:]):  # T = 64 ends on a boundary: the next mini-batch starts from W_T
        np.testing.assert_array_equal(a, b)


@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mlp_reduced(ttt, seed):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=200)
    compare_mlp(ttt, w, make_inputs(w, seed))


@pytest.mark.parametrize("mb", [1, 8, 32])
def test_mlp_mini_batch_sizes(ttt, mb):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=96)
    compare_mlp(ttt, w, make_inputs(w, 3), mini_batch=mb)


def test_mlp_f32_inputs(ttt):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=64, dtype="f32")
    compare_mlp(ttt, w, make_inputs(w, 2))


def test_mlp_auto_picks_split_on_the_8k_workload(ttt):
    """AUTO runs the split tensor-core family on the benchmarked 8k workload."""
    w = WORKLOADS["mlp_8k"]
    assert ttt.mlp_pick_impl(w.B, w.H, w.T, w.d, w.hidden, w.mini_batch, w.dtype) == "tensorcore_split"


@pytest.mark.parametrize("impl", TC_MLP)
@pytest.mark.parametrize("seed", [0, 1, 2])
def test_mlp_full_all_scans(ttt, impl, seed):
    """The full 8k TTT-MLP workload, all 48 scans checked against the oracle, for
    each tensor-core family (seed 0 for the one-CTA family)."""
    if impl == "tensorcore" and seed > 0:
        pytest.skip("the one-CTA family is checked in full on one seed")
    w = WORKLOADS["mlp_8k"]
    compare_mlp(ttt, w, make_inputs(w, seed), impl=impl)


@pytest.mark.parametrize("impl", TC_MLP)
@pytest.mark.parametrize("T", [16, 48, 256, 1024])
@pytest.mark.parametrize("seed", [0, 1])
def test_mlp_tensorcore_vs_oracle(ttt, T, seed, impl):
    """Several chunks, all heads of a small batch, each tensor-core family explicitly."""
    w = WORKLOADS["mlp_8k"].with_shape(B=2, H=3, T=T)
    compare_mlp(ttt, w, make_inputs(w, seed), impl=impl)


def test_mlp_split_matches_one_cta_family(ttt):
    """The two tensor-core families differ only in summation order."""
    w = WORKLOADS["mlp_8k"].with_shape(B=2, H=2, T=1024)
    inp = make_inputs(w, 10)
    a = gpu_mlp(ttt, w, inp, impl="tensorcore_split")
    b = gpu_mlp(ttt, w, inp, impl="tensorcore")
    for name, x, y in zip(("Z", "W1_T", "b1_T", "W2_T", "b2_T"), a, b):
        assert_close(x, y.astype(np.float64), 1e-4, f"{name} split vs one CTA", denom=max(rms(y), 1e-3))


def test_mlp_generic_explicit_on_the_tensorcore_shape(ttt):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=128)
    compare_mlp(ttt, w, make_inputs(w, 4), impl="generic")


@pytest.mark.parametrize("impl", TC_MLP)
def test_mlp_tensorcore_matches_generic(ttt, impl):
    w = WORKLOADS["mlp_8k"].with_shape(B=2, H=2, T=512)
    inp = make_inputs(w, 9)
    tc = gpu_mlp(ttt, w, inp, impl=impl)
    ge = gpu_mlp(ttt, w, inp, impl="generic")
    for name, a, b in zip(("Z", "W1_T", "b1_T", "W2_T", "b2_T"), tc, ge):
        assert_close(a, b.astype(np.float64), 1e-3, f"{name} tensorcore vs generic",
                     denom=max(rms(b), 1e-3))


@pytest.mark.parametrize("impl", TC_MLP)
def test_mlp_tensorcore_continuation(ttt, impl):
    """Two calls split at a mini-batch boundary, the state carried through the
    final-state buffers, equal one call up to rounding."""
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=256)
    inp = make_inputs(w, 5)
    full = gpu_mlp(ttt, w, inp, impl=impl)
    half = w.with_shape(T=128)
    first = {k: (v[:, :, :128].contiguous() if k in ("Q", "K", "V", "eta") else v) for k, v in inp.items()}
    out1 = gpu_mlp(ttt, half, first, impl=impl)
    second = {k: (v[:, :, 128:].contiguous() if k in ("Q", "K", "V", "eta") else v) for k, v in inp.items()}
    for k, o in zip(("W1_0", "b1_0", "W2_0", "b2_0"), out1[1:]):
        second[k] = torch.from_numpy(o)
    out2 = gpu_mlp(ttt, half, second, impl=impl)
    Z = np.concatenate([out1[0], out2[0]], axis=2)
    assert_close(Z, full[0].astype(np.float64), 1e-4, "Z continuation")
    for name, a, b in zip(("W1_T", "b1_T", "W2_T", "b2_T"), out2[1:], full[1:]):
        assert_close(a, b.astype(np.float64), 1e-4, name, denom=max(rms(b), 1e-3))


@pytest.mark.parametrize("impl", TC_MLP)
def test_mlp_tensorcore_is_deterministic(ttt, impl):
    w = WORKLOADS["mlp_8k"].with_shape(B=2, H=2, T=256)
    inp = make_inputs(w, 6)
    a = gpu_mlp(ttt, w, inp, impl=impl)
    b = gpu_mlp(ttt, w, inp, impl=impl)
    for x, y in zip(a, b):
        np.testing.assert_array_equal(x, y)


def test_mlp_host_buffers_end_to_end(ttt):
    """CPU tensors in, CPU tensors out through the public call (the bench's
    end-to-end path), equal to the device-resident call."""
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=128)
    inp = make_inputs(w, 7)
    host = ttt.ttt_mlp_forward(*(inp[k] for k in MLP_KEYS), mini_batch=w.mini_batch, ln_eps=w.ln_eps)
    assert all(o.device.type == "cpu" for o in host)
    dev = gpu_mlp(ttt, w, inp)
    for a, b in zip(host, dev):
        np.testing.assert_array_equal(a.numpy(), b)


@pytest.mark.parametrize("impl", TC_MLP + ["generic"])
def test_mlp_in_place_state(ttt, impl):
    """Final-state buffers that are the initial-state buffers (in-place update)."""
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=2, T=64)
    inp = make_inputs(w, 8)
    ref = gpu_mlp(ttt, w, inp, impl=impl)
    g = to_cuda(inp)
    ttt.ttt_mlp_forward(*(g[k] for k in MLP_KEYS), mini_batch=w.mini_batch, ln_eps=w.ln_eps, impl=impl,
                        W1_T=g["W1_0"], b1_T=g["b1_0"], W2_T=g["W2_0"], b2_T=g["b2_0"])
    torch.cuda.synchronize()
    for name, r in zip(("W1_0", "b1_0", "W2_0", "b2_0"), ref[1:]):
        np.testing.assert_array_equal(g[name].cpu().numpy(), r)


@pytest.mark.parametrize("impl", TC_MLP)
@pytest.mark.parametrize("kw", [dict(T=40), dict(dtype="f32", T=64)])
def test_mlp_tensorcore_unsupported_shapes(ttt, kw, impl):
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=1, **kw)
    with pytest.raises(ttt.TTTError) as ei:
        gpu_mlp(ttt, w, make_inputs(w, 0), impl=impl)
    assert ei.value.status == 6
