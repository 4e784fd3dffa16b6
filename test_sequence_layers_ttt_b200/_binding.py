"""ctypes binding of libttt_b200.so (include/ttt.h).  Argument marshalling only.

Every step of the scan runs in the library's CUDA kernels; this module checks
tensor metadata, allocates outputs through torch when the caller does not pass
them, and forwards raw pointers and the current CUDA stream.  If the inputs
are CPU tensors, the call copies them to the GPU (from pinned memory), runs
the kernels and copies the outputs back: the end-to-end path.

Importing this module raises if the library has not been built: there is no
CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from contextlib import nullcontext as _nullcontext
from typing import Optional, Tuple

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# TTT_B200_LIBRARY may name another build of the same library (the timeline build)
LIB_PATH = os.environ.get("TTT_B200_LIBRARY") or os.path.join(_PKG, "libttt_b200.so")

TTT_BF16, TTT_F32 = 0, 1
TTT_LN_RESIDUAL, TTT_PLAIN = 0, 1
IMPLS = {"auto": 0, "generic": 1, "tensorcore": 2, "tensorcore_split": 3, "tcgen05": 4}
_IMPL_NAMES = {0: "none", 1: "generic", 2: "tensorcore", 3: "tensorcore_split", 4: "tcgen05"}
STATUS = ["TTT_OK", "TTT_ERR_NULL", "TTT_ERR_SHAPE", "TTT_ERR_DTYPE", "TTT_ERR_ALIGN",
          "TTT_ERR_ALIAS", "TTT_ERR_UNSUPPORTED", "TTT_ERR_CUDA", "TTT_ERR_TIMEOUT", "TTT_ERR_WORKSPACE"]


class TTTError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{message} (status {status})")
        self.status = status


if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build the CUDA library first "
        "(python -m test_sequence_layers_ttt_b200.build or __graft_entry__.build())")

lib = ctypes.CDLL(LIB_PATH)
_I, _F, _P = ctypes.c_int, ctypes.c_float, ctypes.c_void_p
lib.ttt_linear_forward.restype = _I
lib.ttt_linear_forward.argtypes = [_I] * 7 + [_F] + [_P] * 11 + [_P]
lib.ttt_linear_forward_impl.restype = _I
lib.ttt_linear_forward_impl.argtypes = [_I] * 7 + [_F] + [_P] * 11 + [_I, _P]
lib.ttt_mlp_forward.restype = _I
lib.ttt_mlp_forward.argtypes = [_I] * 7 + [_F] + [_P] * 15 + [_P]
lib.ttt_mlp_forward_impl.restype = _I
lib.ttt_mlp_forward_impl.argtypes = [_I] * 7 + [_F] + [_P] * 15 + [_I, _P]
lib.ttt_mlp_pick_impl.restype = _I
lib.ttt_mlp_pick_impl.argtypes = [_I] * 7
lib.ttt_status_string.restype = ctypes.c_char_p
lib.ttt_status_string.argtypes = [_I]
lib.ttt_abi_version.restype = _I
lib.ttt_abi_version.argtypes = []
lib.ttt_linear_pick_impl.restype = _I
lib.ttt_linear_pick_impl.argtypes = [_I] * 7
lib.ttt_linear_decode.restype = _I
lib.ttt_linear_decode.argtypes = [_I] * 8 + [_F] + [_P] * 11 + [_P]
lib.ttt_mlp_decode.restype = _I
lib.ttt_mlp_decode.argtypes = [_I] * 8 + [_F] + [_P] * 15 + [_P]
lib.ttt_mlp_decode_impl.restype = _I
lib.ttt_mlp_decode_impl.argtypes = [_I] * 8 + [_F] + [_P] * 15 + [_I, _P]
lib.ttt_linear_backward_workspace_size.restype = ctypes.c_size_t
lib.ttt_linear_backward_workspace_size.argtypes = [_I] * 5
lib.ttt_linear_backward.restype = _I
lib.ttt_linear_backward.argtypes = [_I] * 7 + [_F] + [_P] * 20 + [ctypes.c_size_t, _P]
lib.ttt_linear_backward_static.restype = _I
lib.ttt_linear_backward_static.argtypes = [_I] * 7 + [_F] + [_P] * 19 + [_P]
STATIC_WORKSPACE_BYTES = 32 << 20  # TTT_BACKWARD_STATIC_WORKSPACE_BYTES in include/ttt.h
lib.ttt_prologue_forward.restype = _I
lib.ttt_prologue_forward.argtypes = [_I] * 6 + [_F, _F, _I] + [_P] * 10 + [_P]


def linear_pick_impl(B, H, T, d, mini_batch, qkv_dtype, mode="ln") -> str:
    """Kernel family the library's AUTO dispatch runs for these arguments."""
    code = lib.ttt_linear_pick_impl(B, H, T, d, mini_batch,
                                    TTT_BF16 if qkv_dtype in ("bf16", torch.bfloat16) else TTT_F32,
                                    _mode_code(mode))
    return _IMPL_NAMES[code]


def mlp_pick_impl(B, H, T, d, hidden, mini_batch, qkv_dtype) -> str:
    """Kernel family the library's AUTO dispatch runs for these TTT-MLP arguments."""
    code = lib.ttt_mlp_pick_impl(B, H, T, d, hidden, mini_batch,
                                 TTT_BF16 if qkv_dtype in ("bf16", torch.bfloat16) else TTT_F32)
    return _IMPL_NAMES[code]


def status_string(status: int) -> str:
    return lib.ttt_status_string(status).decode()


def _check(status: int):
    if status != 0:
        raise TTTError(status, status_string(status))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.bfloat16:
        return TTT_BF16
    if t.dtype == torch.float32:
        return TTT_F32
    raise TypeError(f"Q/K/V must be bf16 or fp32, got {t.dtype}")


def _mode_code(mode) -> int:
    if mode in ("ln", "ln_residual", TTT_LN_RESIDUAL):
        return TTT_LN_RESIDUAL
    if mode in ("plain", TTT_PLAIN):
        return TTT_PLAIN
    raise ValueError(f"unknown mode {mode!r}")


def _stream_handle(device: torch.device, stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream(device)
    handle = stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream)
    return ctypes.c_void_p(handle)


def _launch_stream(device: torch.device, stream):
    """The stream a call enqueues on, as a torch stream object."""
    if stream is None:
        return torch.cuda.current_stream(device)
    if isinstance(stream, torch.cuda.Stream):
        return stream
    return torch.cuda.ExternalStream(int(getattr(stream, "cuda_stream", stream)), device=device)


class _HostRoundTrip:
    """Moves CPU inputs to the GPU and device outputs back (end-to-end path).

    The copies in, the launch and the copies back are all enqueued on the one
    stream the call launches on, so stream order alone makes the kernel see its
    inputs and the copies back see its outputs."""

    def __init__(self, tensors, stream=None):
        self.on_host = any(t is not None and t.device.type == "cpu" for t in tensors)
        self.device = torch.device("cuda", torch.cuda.current_device()) if self.on_host else None
        self.stream = _launch_stream(self.device, stream) if self.on_host else None

    def to_device(self, t):
        if t is None or not self.on_host:
            return t
        if t.device.type != "cpu":
            return t
        src = t if t.is_pinned() else t.pin_memory()
        with torch.cuda.stream(self.stream):
            return src.to(self.device, non_blocking=True)

    def to_host(self, outs):
        if not self.on_host:
            return outs
        host = []
        with torch.cuda.stream(self.stream):
            for o in outs:
                if o is None:
                    host.append(None)
                    continue
                h = torch.empty(o.shape, dtype=o.dtype, pin_memory=True)
                h.copy_(o, non_blocking=True)
                host.append(h)
        self.stream.synchronize()
        return tuple(host)


_STREAMS = {}


def _side_streams(dev: torch.device, n: int):
    key = (dev.index, n)
    if key not in _STREAMS:
        _STREAMS[key] = [torch.cuda.Stream(device=dev) for _ in range(n)]
    return _STREAMS[key]


def _head_groups(B: int, H: int, n: int):
    """(batch, first head, end head) groups of about B*H/n scans each."""
    per = max(1, -(-(B * H) // n))
    return [(b, h0, min(H, h0 + per)) for b in range(B) for h0 in range(0, H, per)]


def _pinned(t):
    return None if t is None else (t if t.is_pinned() else t.pin_memory())


def _host_pipeline(device_call, per_scan: dict, per_head: dict, out_shapes: dict, n_groups: int = 8):
    """End-to-end path for host tensors: the (batch, head) scans are independent,
    so they are cut into groups, and each group's copies in, scan and copies out
    run on their own stream; one group's transfers overlap the others' scans and
    the two copy directions overlap each other.  Results land in pinned host
    tensors; the call returns when every copy back has finished."""
    dev = torch.device("cuda", torch.cuda.current_device())
    any_t = next(t for t in per_scan.values() if t is not None)
    B, H = any_t.shape[:2]
    per_scan = {k: _pinned(t) for k, t in per_scan.items()}
    per_head = {k: _pinned(t) for k, t in per_head.items()}
    outs = {k: (None if shp is None else torch.empty(shp, dtype=torch.float32, pin_memory=True))
            for k, shp in out_shapes.items()}
    groups = _head_groups(B, H, n_groups)
    streams = _side_streams(dev, min(n_groups, len(groups)))
    current = torch.cuda.current_stream(dev)
    for s in streams:
        s.wait_stream(current)
    for i, (b, h0, h1) in enumerate(groups):
        s = streams[i % len(streams)]
        with torch.cuda.stream(s):
            args = {k: (None if t is None else t[b:b + 1, h0:h1].to(dev, non_blocking=True))
                    for k, t in per_scan.items()}
            args.update({k: (None if t is None else t[h0:h1].to(dev, non_blocking=True))
                         for k, t in per_head.items()})
            res = device_call(args, s)
            for (k, host), r in zip(outs.items(), res):
                if host is not None:
                    host[b:b + 1, h0:h1].copy_(r, non_blocking=True)
    for s in streams:
        s.synchronize()
    return tuple(outs.values())


def _on_host(*ts) -> bool:
    return all(t is None or t.device.type == "cpu" for t in ts)


def ttt_linear_forward(Q, K, V, eta, W0, b0=None, ln_gamma=None, ln_beta=None, *,
                       mini_batch: int = 16, mode="ln", ln_eps: float = 1e-6, impl: str = "auto",
                       Z=None, W_T=None, b_T=None, stream=None
                       ) -> Tuple[torch.Tensor, torch.Tensor, Optional[torch.Tensor]]:
    """TTT-Linear forward scan (see include/ttt.h).  Returns (Z, W_T, b_T).
    Host (CPU) tensors in, host tensors out when every input is on the host."""
    if (_on_host(Q, K, V, eta, W0, b0, ln_gamma, ln_beta) and Z is None and W_T is None and b_T is None
            and stream is None and Q.dim() == 4 and Q.shape[0] * Q.shape[1] > 1 and Q.shape[2] > 0):
        B, H, T, d = Q.shape
        plain = _mode_code(mode) == TTT_PLAIN

        def run(a, s):
            return ttt_linear_forward(a["Q"], a["K"], a["V"], a["eta"], a["W0"], a["b0"], a["ln_gamma"],
                                      a["ln_beta"], mini_batch=mini_batch, mode=mode, ln_eps=ln_eps,
                                      impl=impl, stream=s)

        return _host_pipeline(run, dict(Q=Q, K=K, V=V, eta=eta, W0=W0, b0=b0),
                              dict(ln_gamma=ln_gamma, ln_beta=ln_beta),
                              dict(Z=(B, H, T, d), W_T=(B, H, d, d), b_T=None if plain else (B, H, d)))
    rt = _HostRoundTrip([Q, K, V, eta, W0], stream)
    if rt.on_host:
        stream = rt.stream
    Q, K, V, eta, W0, b0, ln_gamma, ln_beta = (
        rt.to_device(x) for x in (Q, K, V, eta, W0, b0, ln_gamma, ln_beta))
    B, H, T, d = Q.shape
    m = _mode_code(mode)
    for name, t in (("Q", Q), ("K", K), ("V", V), ("eta", eta), ("W0", W0), ("b0", b0),
                    ("ln_gamma", ln_gamma), ("ln_beta", ln_beta)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if K.shape != Q.shape or V.shape != Q.shape or K.dtype != Q.dtype or V.dtype != Q.dtype:
        raise ValueError("Q, K, V must share shape and dtype")
    if tuple(eta.shape) != (B, H, T) or tuple(W0.shape) != (B, H, d, d):
        raise ValueError("eta must be [B,H,T] and W0 [B,H,d,d]")
    dev = Q.device
    with torch.cuda.stream(rt.stream) if rt.on_host else _nullcontext():
        if Z is None:
            Z = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
        if W_T is None:
            W_T = torch.empty((B, H, d, d), dtype=torch.float32, device=dev)
        if b_T is None and m == TTT_LN_RESIDUAL:
            b_T = torch.empty((B, H, d), dtype=torch.float32, device=dev)
    st = lib.ttt_linear_forward_impl(
        B, H, T, d, int(mini_batch), _dtype_code(Q), m, float(ln_eps), _ptr(Q), _ptr(K), _ptr(V),
        _ptr(eta), _ptr(W0), _ptr(b0), _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z), _ptr(W_T),
        _ptr(b_T), IMPLS[impl], _stream_handle(dev, stream))
    _check(st)
    return rt.to_host((Z, W_T, b_T))


def ttt_linear_decode(Q, K, V, eta, W, b, W_mb, b_mb, ln_gamma=None, ln_beta=None, *, pos0: int,
                      mini_batch: int = 16, mode="ln", ln_eps: float = 1e-6, Z=None, stream=None
                      ) -> torch.Tensor:
    """TTT-Linear decode (see include/ttt.h): the scan continued by T tokens from
    position pos0 of a mini-batch.  W, b (running state) and W_mb, b_mb (the
    current mini-batch's start state) are CUDA tensors updated in place; the
    next call's pos0 is (pos0 + T) % mini_batch.  Returns Z."""
    m = _mode_code(mode)
    B, H, T, d = Q.shape
    for name, t in (("Q", Q), ("K", K), ("V", V), ("eta", eta), ("W", W), ("b", b), ("W_mb", W_mb),
                    ("b_mb", b_mb), ("ln_gamma", ln_gamma), ("ln_beta", ln_beta)):
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if K.shape != Q.shape or V.shape != Q.shape or K.dtype != Q.dtype or V.dtype != Q.dtype:
        raise ValueError("Q, K, V must share shape and dtype")
    if tuple(eta.shape) != (B, H, T) or tuple(W.shape) != (B, H, d, d) or tuple(W_mb.shape) != (B, H, d, d):
        raise ValueError("eta must be [B,H,T], W and W_mb [B,H,d,d]")
    for name, t in (("W", W), ("b", b), ("W_mb", W_mb), ("b_mb", b_mb), ("eta", eta)):
        if t is not None and t.dtype != torch.float32:
            raise TypeError(f"{name} must be float32")
    dev = Q.device
    if Z is None:
        Z = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
    st = lib.ttt_linear_decode(
        B, H, T, d, int(mini_batch), int(pos0), _dtype_code(Q), m, float(ln_eps), _ptr(Q), _ptr(K), _ptr(V),
        _ptr(eta), _ptr(W), _ptr(b), _ptr(W_mb), _ptr(b_mb), _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z),
        _stream_handle(dev, stream))
    _check(st)
    return Z


def ttt_mlp_decode(Q, K, V, eta, W1, b1, W2, b2, W1_mb, b1_mb, W2_mb, b2_mb, ln_gamma, ln_beta, *,
                   pos0: int, mini_batch: int = 16, ln_eps: float = 1e-6, impl: str = "auto", Z=None,
                   stream=None) -> torch.Tensor:
    """TTT-MLP decode (see include/ttt.h): the scan continued by T tokens from
    position pos0 of a mini-batch.  The running state (W1, b1, W2, b2) and the
    mini-batch start state (W1_mb, ...) are CUDA tensors updated in place.
    Returns Z."""
    B, H, T, d = Q.shape
    state = (W1, b1, W2, b2, W1_mb, b1_mb, W2_mb, b2_mb)
    for name, t in (("Q", Q), ("K", K), ("V", V), ("eta", eta), ("ln_gamma", ln_gamma), ("ln_beta", ln_beta),
                    *zip(("W1", "b1", "W2", "b2", "W1_mb", "b1_mb", "W2_mb", "b2_mb"), state)):
        if t is None or not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if K.shape != Q.shape or V.shape != Q.shape or K.dtype != Q.dtype or V.dtype != Q.dtype:
        raise ValueError("Q, K, V must share shape and dtype")
    hidden = W1.shape[-1]
    shapes = ((B, H, d, hidden), (B, H, hidden), (B, H, hidden, d), (B, H, d)) * 2
    if tuple(eta.shape) != (B, H, T) or any(tuple(t.shape) != sh for t, sh in zip(state, shapes)):
        raise ValueError("eta must be [B,H,T]; W1 [B,H,d,hid], b1 [B,H,hid], W2 [B,H,hid,d], b2 [B,H,d]")
    if any(t.dtype != torch.float32 for t in (eta, *state)):
        raise TypeError("eta and the state must be float32")
    dev = Q.device
    if Z is None:
        Z = torch.empty((B, H, T, d), dtype=torch.float32, device=dev)
    st = lib.ttt_mlp_decode_impl(
        B, H, T, d, hidden, int(mini_batch), int(pos0), _dtype_code(Q), float(ln_eps), _ptr(Q), _ptr(K), _ptr(V),
        _ptr(eta), *(_ptr(t) for t in state), _ptr(ln_gamma), _ptr(ln_beta), _ptr(Z), IMPLS[impl],
        _stream_handle(dev, stream))
    _check(st)
    return Z


def ttt_mlp_forward(Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, ln_gamma, ln_beta, *,
                    mini_batch: int = 16, ln_eps: float = 1e-6, impl: str = "auto", Z=None,
                    W1_T=None, b1_T=None, W2_T=None, b2_T=None, stream=None):
    """TTT-MLP forward scan (see include/ttt.h).  Returns (Z, W1_T, b1_T, W2_T, b2_T).
    Host (CPU) tensors in, host tensors out when every input is on the host."""
    if (_on_host(Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, ln_gamma, ln_beta)
            and all(o is None for o in (Z, W1_T, b1_T, W2_T, b2_T)) and stream is None and Q.dim() == 4
            and Q.shape[0] * Q.shape[1] > 1 and Q.shape[2] > 0):
        B, H, T, d = Q.shape
        hid = W1_0.shape[-1]

        def run(a, s):
            return ttt_mlp_forward(a["Q"], a["K"], a["V"], a["eta"], a["W1_0"], a["b1_0"], a["W2_0"],
                                   a["b2_0"], a["ln_gamma"], a["ln_beta"], mini_batch=mini_batch,
                                   ln_eps=ln_eps, impl=impl, stream=s)

        return _host_pipeline(run, dict(Q=Q, K=K, V=V, eta=eta, W1_0=W1_0, b1_0=b1_0, W2_0=W2_0, b2_0=b2_0),
                              dict(ln_gamma=ln_gamma, ln_beta=ln_beta),
                              dict(Z=(B, H, T, d), W1_T=(B, H, d, hid), b1_T=(B, H, hid),
                                   W2_T=(B, H, hid, d), b2_T=(B, H, d)))
    rt = _HostRoundTrip([Q, K, V, eta, W1_0], stream)
    if rt.on_host:
        stream = rt.stream
    Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, ln_gamma, ln_beta = (
        rt.to_device(x) for x in (Q, K, V, eta, W1_0, b1_0, W2_0, b2_0, ln_gamma, ln_beta))
    B, H, T, d = Q.shape
    hid = W1_0.shape[-1]
    for name, t in (("Q", Q), ("K", K), ("V", V), ("eta", eta), ("W1_0", W1_0), ("b1_0", b1_0),
                    ("W2_0", W2_0), ("b2_0", b2_0), ("ln_gamma", ln_gamma), ("ln_beta", ln_beta)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    dev = Q.device
    f32 = dict(dtype=torch.float32, device=dev)
    with torch.cuda.stream(rt.stream) if rt.on_host else _nullcontext():
        Z = torch.empty((B, H, T, d), **f32) if Z is None else Z
        W1_T = torch.empty((B, H, d, hid), **f32) if W1_T is None else W1_T
        b1_T = torch.empty((B, H, hid), **f32) if b1_T is None else b1_T
        W2_T = torch.empty((B, H, hid, d), **f32) if W2_T is None else W2_T
        b2_T = torch.empty((B, H, d), **f32) if b2_T is None else b2_T
    st = lib.ttt_mlp_forward_impl(
        B, H, T, d, hid, int(mini_batch), _dtype_code(Q), float(ln_eps), _ptr(Q), _ptr(K),
        _ptr(V), _ptr(eta), _ptr(W1_0), _ptr(b1_0), _ptr(W2_0), _ptr(b2_0), _ptr(ln_gamma),
        _ptr(ln_beta), _ptr(Z), _ptr(W1_T), _ptr(b1_T), _ptr(W2_T), _ptr(b2_T), IMPLS[impl],
        _stream_handle(dev, stream))
    _check(st)
    return rt.to_host((Z, W1_T, b1_T, W2_T, b2_T))


def linear_backward_workspace_size(B: int, H: int, T: int, d: int, mini_batch: int) -> int:
    """Bytes of device workspace ttt_linear_backward needs (see include/ttt.h)."""
    return int(lib.ttt_linear_backward_workspace_size(B, H, T, d, mini_batch))


def ttt_linear_backward(Q, K, V, eta, W0, b0, ln_gamma, ln_beta, dZ, dW_T=None, db_T=None, *,
                        mini_batch: int = 16, mode="ln", ln_eps: float = 1e-6, workspace=None, stream=None):
    """TTT-Linear layer backward (see include/ttt.h): gradients of
    sum(Z dZ) + sum(W_T dW_T) + sum(b_T db_T) with respect to the forward inputs.
    Returns (dQ, dK, dV, deta, dW0, db0, dgamma, dbeta), fp32 CUDA tensors.  The
    workspace (a CUDA byte tensor) is allocated here when not given."""
    B, H, T, d = Q.shape
    named = (("Q", Q), ("K", K), ("V", V), ("eta", eta), ("W0", W0), ("b0", b0), ("ln_gamma", ln_gamma),
             ("ln_beta", ln_beta), ("dZ", dZ), ("dW_T", dW_T), ("db_T", db_T))
    for name, t in named:
        if t is not None and (not t.is_cuda or not t.is_contiguous()):
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if K.shape != Q.shape or V.shape != Q.shape or K.dtype != Q.dtype or V.dtype != Q.dtype:
        raise ValueError("Q, K, V must share shape and dtype")
    if tuple(dZ.shape) != (B, H, T, d) or dZ.dtype != torch.float32:
        raise ValueError("dZ must be float32 [B,H,T,d]")
    dev = Q.device
    f32 = dict(dtype=torch.float32, device=dev)
    dQ, dK, dV = (torch.empty((B, H, T, d), **f32) for _ in range(3))
    deta = torch.empty((B, H, T), **f32)
    dW0 = torch.empty((B, H, d, d), **f32)
    db0 = torch.empty((B, H, d), **f32)
    dgamma = torch.empty((H, d), **f32)
    dbeta = torch.empty((H, d), **f32)
    need = linear_backward_workspace_size(B, H, T, d, mini_batch)
    if workspace is None:
        workspace = torch.empty(max(need, 16), dtype=torch.uint8, device=dev)
    st = lib.ttt_linear_backward(
        B, H, T, d, int(mini_batch), _dtype_code(Q), _mode_code(mode), float(ln_eps), _ptr(Q), _ptr(K), _ptr(V),
        _ptr(eta), _ptr(W0), _ptr(b0), _ptr(ln_gamma), _ptr(ln_beta), _ptr(dZ), _ptr(dW_T), _ptr(db_T),
        _ptr(dQ), _ptr(dK), _ptr(dV), _ptr(deta), _ptr(dW0), _ptr(db0), _ptr(dgamma), _ptr(dbeta),
        _ptr(workspace), ctypes.c_size_t(workspace.numel() * workspace.element_size()),
        _stream_handle(dev, stream))
    _check(st)
    return dQ, dK, dV, deta, dW0, db0, dgamma, dbeta


def ttt_prologue_forward(x, theta_q, theta_k, theta_v, theta_lr, b_lr, *, pos0: int = 0,
                         eta_base: float = 1.0, rope_base: float = 10000.0, rotary: bool = True,
                         stream=None):
    """The layer's prologue (see include/ttt.h): Q, K, V [B,H,T,d] bf16 and eta
    [B,H,T] fp32 from x [B,T,d_model] bf16 and the bf16 weights."""
    B, T, dm = x.shape
    H, _, d = theta_q.shape
    for name, t in (("x", x), ("theta_q", theta_q), ("theta_k", theta_k), ("theta_v", theta_v),
                    ("theta_lr", theta_lr), ("b_lr", b_lr)):
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous CUDA tensor")
    if any(t.dtype != torch.bfloat16 for t in (x, theta_q, theta_k, theta_v, theta_lr)) or b_lr.dtype != torch.float32:
        raise TypeError("x and the weights must be bfloat16, b_lr float32")
    dev = x.device
    Q, K, V = (torch.empty((B, H, T, d), dtype=torch.bfloat16, device=dev) for _ in range(3))
    eta = torch.empty((B, H, T), dtype=torch.float32, device=dev)
    st = lib.ttt_prologue_forward(B, T, H, d, dm, int(pos0), float(eta_base), float(rope_base), int(bool(rotary)),
                                  _ptr(x), _ptr(theta_q), _ptr(theta_k), _ptr(theta_v), _ptr(theta_lr), _ptr(b_lr),
                                  _ptr(Q), _ptr(K), _ptr(V), _ptr(eta), _stream_handle(dev, stream))
    _check(st)
    return Q, K, V, eta
