"""Clock64 timeline of one TTT-Linear tensor-core launch: where a chunk step's
cycles go, per warp role.

Builds the library with the timeline stamps compiled in
(libttt_b200_timeline.so), runs one 1.3B-shape launch (B2 H32 T32768 d64,
bf16) of the chosen family, and prints, from CTA 0's stamps over 32
consecutive chunk steps of mid-sequence: the period of every role, the median
time between the role's stamped points, and the median time from the chain's
hand-off of chunk c to each consumer's pick-up.

    python -m test_sequence_layers_ttt_b200.timeline [tensorcore]

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
    main(sys.argv[1] if len(sys.argv) > 1 else "tensorcore")
