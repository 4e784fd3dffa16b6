"""Seeded synthetic workloads for the TTT forward scan.

This module only draws random numbers and lays them out; it holds none of the
scan's arithmetic.  The same arrays feed the float64 oracle and the CUDA
library, so both sides see identical bits.

Workloads follow the shapes and distributions stated for the TTT layer
("Learning to (Learn at Test Time): RNNs with Expressive Hidden States"):
TTT-Linear at the 125M and 1.3B layer shapes (head dim 64, mini-batch 16,
contexts up to 32k), a small fp32 case, the Theorem-1 case (linear f, W0 = 0,
eta = 1/2, batch GD) and a TTT-MLP layer (64 -> 256 -> 64).

Draw order for one seed (CPU ``torch.Generator``, fp32): u (for eta), Q, K, V,
then W0 (or W1, W2), then gamma, beta.  Per-head parameters (W0, gamma, beta)
are drawn once per head and shared by every batch row, as a layer's initial
weights are.  Q, K, V are rounded to bf16 (round-to-nearest-even) for the bf16
workloads; the rounded values are what both sides consume.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, replace
from typing import Dict, Optional

import torch

MODE_LN_RESIDUAL = 0  # f(x) = x + LN(x W + b)
MODE_PLAIN = 1        # f(x) = x W  (the Theorem-1 setting)


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "linear" or "mlp"
    B: int
    H: int
    T: int
    d: int
    mini_batch: int
    dtype: str           # "f32" or "bf16" (dtype of Q, K, V)
    mode: int = MODE_LN_RESIDUAL
    hidden: int = 0      # MLP hidden width
    init: str = "lm"     # parameter recipe, see make_inputs
    ln_eps: float = 1e-6

    def with_shape(self, **kw) -> "Workload":
        return replace(self, **kw)

    @property
    def head_tokens(self) -> int:
        return self.B * self.H * self.T


WORKLOADS: Dict[str, Workload] = {
    # TTT-Linear single layer, fp32: B=1, H=2, d=16, T=64, b=16.
    "linear_tiny_f32": Workload("linear_tiny_f32", "linear", 1, 2, 64, 16, 16, "f32", init="unit"),
    # Theorem 1: f(x) = x W, W0 = 0, eta = 1/2, one mini-batch over all tokens.
    "theorem1_f32": Workload("theorem1_f32", "linear", 2, 4, 1024, 64, 1024, "f32",
                             mode=MODE_PLAIN, init="theorem1"),
    # 125M-class TTT-Linear layer: B=8, H=12, d=64, T=2048, b=16, bf16 Q/K/V.
    "linear_125m_2k": Workload("linear_125m_2k", "linear", 8, 12, 2048, 64, 16, "bf16", init="lm"),
    # 1.3B-class TTT-Linear layer, 32k context: B=2, H=32, d=64, T=32768, b=16.
    "linear_1p3b_32k": Workload("linear_1p3b_32k", "linear", 2, 32, 32768, 64, 16, "bf16", init="lm"),
    # Decode on the 1.3B-class layer: the stream of B=2 sequences x H=32 heads
    # continued one token per step; T is the number of tokens generated.
    "decode_1p3b": Workload("decode_1p3b", "linear", 2, 32, 256, 64, 16, "bf16", init="lm"),
    # Decode on the TTT-MLP layer: B=4 x H=12 streams, one token per step.
    "decode_mlp_8k": Workload("decode_mlp_8k", "mlp", 4, 12, 256, 64, 16, "bf16", hidden=256, init="mlp"),
    # TTT-MLP layer: B=4, H=12, d=64, 64 -> 256 -> 64, T=8192, b=16.
    "mlp_8k": Workload("mlp_8k", "mlp", 4, 12, 8192, 64, 16, "bf16", hidden=256, init="mlp"),
}


def _normal(gen: torch.Generator, shape, std: float) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32) * std


def make_inputs(w: Workload, seed: int) -> Dict[str, Optional[torch.Tensor]]:
    """Return the CPU tensors of one seeded instance of workload ``w``.

    Keys: Q, K, V ([B,H,T,d], bf16 or fp32), eta ([B,H,T] fp32), gamma, beta
    ([H,d] fp32) and, for TTT-Linear, W0 ([B,H,d,d], W[in][out]) and b0
    ([B,H,d]); for TTT-MLP, W1_0 ([B,H,d,hidden]), b1_0, W2_0
    ([B,H,hidden,d]), b2_0.  All parameter tensors are fp32.
    """
    gen = torch.Generator(device="cpu")
    gen.manual_seed(seed)
    B, H, T, d = w.B, w.H, w.T, w.d
    qkv_std = 1.0 / math.sqrt(d)

    u = torch.randn(B, H, T, generator=gen, dtype=torch.float32)
    if w.init == "theorem1":
        eta = torch.full((B, H, T), 0.5, dtype=torch.float32)
    else:
        # token-dependent inner learning rate eta_t = sigmoid(u_t) / d
        eta = torch.sigmoid(u) / d

    Q = _normal(gen, (B, H, T, d), qkv_std)
    K = _normal(gen, (B, H, T, d), qkv_std)
    V = _normal(gen, (B, H, T, d), qkv_std)
    if w.dtype == "bf16":
        Q, K, V = (x.to(torch.bfloat16) for x in (Q, K, V))
    elif w.dtype != "f32":
        raise ValueError(f"unknown dtype {w.dtype}")

    out: Dict[str, Optional[torch.Tensor]] = {"Q": Q, "K": K, "V": V, "eta": eta}

    def per_head(x: torch.Tensor) -> torch.Tensor:
        return x.unsqueeze(0).expand(B, *x.shape).contiguous()

    if w.kind == "linear":
        if w.init == "theorem1":
            W0 = torch.zeros(H, d, d)
        elif w.init == "unit":
            W0 = _normal(gen, (H, d, d), 1.0 / math.sqrt(d))
        elif w.init == "lm":
            W0 = _normal(gen, (H, d, d), 0.02)
        else:
            raise ValueError(w.init)
        out["W0"] = per_head(W0)
        out["b0"] = torch.zeros(B, H, d)
    elif w.kind == "mlp":
        h = w.hidden
        out["W1_0"] = per_head(_normal(gen, (H, d, h), 1.0 / math.sqrt(d)))
        out["b1_0"] = torch.zeros(B, H, h)
        out["W2_0"] = per_head(_normal(gen, (H, h, d), 1.0 / math.sqrt(h)))
        out["b2_0"] = torch.zeros(B, H, d)
    else:
        raise ValueError(w.kind)

    if w.init == "lm":
        gamma = 1.0 + _normal(gen, (H, d), 0.02)
        beta = _normal(gen, (H, d), 0.02)
    else:
        gamma = torch.ones(H, d)
        beta = torch.zeros(H, d)
    out["gamma"] = gamma
    out["beta"] = beta
    return out


def select_heads(inp: Dict[str, Optional[torch.Tensor]], pairs) -> Dict[str, Optional[torch.Tensor]]:
    """Gather the (b, h) pairs in ``pairs`` into a B'=1, H'=len(pairs) instance.

    Every (b, h) scan is independent, so a subset of pairs is itself a valid
    instance; gamma/beta follow their head.
    """
    bs = torch.tensor([p[0] for p in pairs])
    hs = torch.tensor([p[1] for p in pairs])
    sel = {}
    for k, x in inp.items():
        if x is None:
            sel[k] = None
        elif k in ("gamma", "beta"):
            sel[k] = x[hs].contiguous()
        else:
            sel[k] = x[bs, hs].unsqueeze(0).contiguous()
    return sel
