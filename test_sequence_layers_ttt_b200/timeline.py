"""Clock64 timeline of one TTT-Linear tensor-core launch: where a chunk step's
cycles go, per warp role.

Builds the library with the timeline stamps compiled in
(libttt_b200_timeline.so), runs one 1.3B-shape launch (B2 H32 T32768 d64,
bf16) of the chosen family, and prints, from CTA 0's stamps over 32
consecutive chunk steps of mid-sequence: the period of every role, the median
time between the role's stamped points, and the median time from the chain's
hand-off of chunk c to each consumer's pick-up.

    python -m test_sequence_layers_ttt_b200.timeline [tensorcore]
    python -m test_sequence_layers_ttt_b200.timeline backward   # the layer backward's reverse sweep

Needs a GPU.  The stamps perturb the kernel a little (one clock read and one
store per point, CTA 0 only).
"""
from __future__ import annotations

import ctypes
import os
import sys

import numpy as np

ROLES = {
    "tensorcore": (0, ["CH", "WP", "OW", "PR", "PA", "PB"], {
        "CH": ["top", "chain mma", "stats barrier", "G formed", "E buffer free", "E handed off", "next inputs",
               "next P in"],
        "WP": ["top", "E in", "update done", "split done", "P slot free", "P handed off", "W slot free",
               "W handed off"],
        "OW": ["top", "W in", "QW formed + L frags in", "E in", "correction done", "stats barrier", "-",
               "stored"],
        "PR": ["top", "stage free"],
        "PA": ["top", "stage in", "slot free", "done"],
        "PB": ["top", "stage in", "slot free", "done"],
    }),
}
N_ROLES, N_CHUNKS, N_EVENTS, FIRST = 8, 32, 8, 1024

# The layer backward's reverse sweep (one CTA per (batch, head), all threads in step): stamp k of a
# mini-batch after the phase named here, in the order they run.
BACKWARD_POINTS = [
    (14, "commit of the prefetched inputs"), (15, "next mini-batch's loads issued"), (0, "barrier"),
    (1, "forward recomputed (2 products, 1 row pass) + Zb products"), (2, "output LayerNorm rows"),
    (3, "dgamma/dbeta; dQ = dZ; dZb (row pass)"), (4, "dZb products (dQ, dW_prev, dG, -X dW) + db_prev"),
    (5, "dA product"), (6, "dA mask; dEG; dG += e dEG"), (7, "de rows"), (8, "tmp = e G; dP = dA e"),
    (9, "dX, dQ products; dW_prev += dW; dG row sums"), (10, "row pass: dGx, dR, dY"),
    (11, "dgamma/dbeta; dX += dR; dV"), (12, "dY products + db_prev"), (13, "stores of dQ, dK, deta; swap"),
]


def backward() -> None:
    """The reverse sweep's per-mini-batch phases (1.3B shape, CTA 0, mini-batches 1024..1055 of the
    sweep)."""
    from test_sequence_layers_ttt_b200 import build as lib_build
    os.environ["TTT_B200_LIBRARY"] = lib_build.build(timeline=True)
    import torch
    from test_sequence_layers_ttt_b200 import _binding as ttt
    from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs

    w = WORKLOADS["linear_1p3b_32k"]
    g = {k: v.cuda() for k, v in make_inputs(w, 0).items()}
    gen = torch.Generator().manual_seed(0)
    dZ = torch.randn((w.B, w.H, w.T, w.d), generator=gen).cuda()
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    for _ in range(2):
        ttt.ttt_linear_backward(*(g[k] for k in keys), dZ, None, None, mini_batch=16, ln_eps=w.ln_eps)
    torch.cuda.synchronize()
    buf = np.zeros((N_ROLES, N_CHUNKS, N_EVENTS), dtype=np.int64)
    fn = ttt.lib.ttt_debug_timeline
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int, ctypes.c_void_p]
    st = fn(1, buf.ctypes.data)
    if st != 0:
        raise RuntimeError(f"ttt_debug_timeline failed with status {st}")
    at = lambda k: buf[k >> 3, :, k & 7].astype(np.float64)
    period = np.median(np.diff(at(0)))
    print(f"backward reverse sweep: CTA 0, mini-batches {FIRST}..{FIRST + N_CHUNKS - 1} of the sweep, "
          f"SM cycles (median)")
    print(f"  period per mini-batch {period:.0f}")
    # each point's interval starts at the point before it; the commit's at the end (13) of the
    # previous mini-batch
    order = [k for k, _ in BACKWARD_POINTS]
    for i, (k, label) in enumerate(BACKWARD_POINTS):
        start = at(13)[:-1] if i == 0 else at(order[i - 1])[1:]
        print(f"  {np.median(at(k)[1:] - start):7.0f}  {label}")


def main(family: str = "tensorcore") -> None:
    from test_sequence_layers_ttt_b200 import build as lib_build
    os.environ["TTT_B200_LIBRARY"] = lib_build.build(timeline=True)
    import torch
    from test_sequence_layers_ttt_b200 import _binding as ttt
    from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs

    which, roles, events = ROLES[family]
    w = WORKLOADS["linear_1p3b_32k"]
    g = {k: v.cuda() for k, v in make_inputs(w, 0).items()}
    keys = ("Q", "K", "V", "eta", "W0", "b0", "gamma", "beta")
    for _ in range(2):
        ttt.ttt_linear_forward(*(g[k] for k in keys), impl=family)
    torch.cuda.synchronize()
    buf = np.zeros((N_ROLES, N_CHUNKS, N_EVENTS), dtype=np.int64)
    fn = ttt.lib.ttt_debug_timeline
    fn.restype = ctypes.c_int
    fn.argtypes = [ctypes.c_int, ctypes.c_void_p]
    st = fn(which, buf.ctypes.data)
    if st != 0:
        raise RuntimeError(f"ttt_debug_timeline failed with status {st}")
    clk = torch.cuda.get_device_properties(0).clock_rate if hasattr(torch.cuda.get_device_properties(0),
                                                                   "clock_rate") else None
    print(f"family {family}: CTA 0, chunk steps {FIRST}..{FIRST + N_CHUNKS - 1}, SM cycles (median over steps)")
    for r, name in enumerate(roles):
        ev = events[name]
        stamps = buf[r, :, :len(ev)].astype(np.float64)
        if not stamps[:, 0].any():
            continue
        period = np.median(np.diff(stamps[:, 0]))
        parts = []
        for e in range(1, len(ev)):
            d = stamps[:, e] - stamps[:, e - 1]
            parts.append(f"{ev[e]} +{np.median(d):.0f}")
        print(f"  {name:3s} period {period:6.0f}: " + ", ".join(parts))
    # hand-off latencies from the chain
    ch = buf[0].astype(np.float64)
    if family == "tensorcore":
        wp = buf[1].astype(np.float64)
        # E_c handed off (CH ev5 of c) -> picked up by WP iteration j = c + 1 (ev1, indexed j)
        d = wp[1:, 1] - ch[:-1, 5]
        print(f"  E_c hand-off -> WP pick-up: {np.median(d):.0f}")
        # P_{j+1} handed off by WP iteration j (ev5, indexed j) -> CH load_inputs(j+1) done (ev7 of chunk j)
        d = ch[:, 7] - wp[:, 5]
        print(f"  P hand-off -> CH pick-up (same index): {np.median(d):.0f}")
    if clk:
        print(f"  (SM clock {clk / 1e3:.0f} MHz nominal)")


if __name__ == "__main__":
    if len(sys.argv) > 1 and sys.argv[1] == "backward":
        backward()
    else:
        main(sys.argv[1] if len(sys.argv) > 1 else "tensorcore")
