"""Write the oracle regression fixture linear_tiny_f32_seed0.txt.

Calls only the oracle and the seeded input generator.  Re-run after a change
to the oracle's arithmetic that the pages justify, and say which passage in
the commit message.
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from test_sequence_layers_ttt_b200.inputs import WORKLOADS, make_inputs  # noqa: E402


def main():
    w = WORKLOADS["linear_tiny_f32"]
    inp = make_inputs(w, 0)
    Z, W_T, b_T = oracle.ttt_linear(inp["Q"], inp["K"], inp["V"], inp["eta"], inp["W0"],
                                    inp["b0"], inp["gamma"], inp["beta"], w.mini_batch)
    idx = np.random.default_rng(1234).choice(Z.size, 48, replace=False)
    idx.sort()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "linear_tiny_f32_seed0.txt")
    with open(out, "w") as fh:
        fh.write("# Oracle regression values: TTT-Linear, B=1 H=2 T=64 d=16 b=16, fp32 inputs,\n")
        fh.write("# seed 0 (test_sequence_layers_ttt_b200.inputs).  Written by make_golden.py\n")
        fh.write("# from the float64 oracle only.  Z_index are flat indices into Z[B,H,T,d].\n")
        fh.write("Z_index " + " ".join(str(int(i)) for i in idx) + "\n")
        fh.write("Z " + " ".join(repr(float(x)) for x in Z.reshape(-1)[idx]) + "\n")
        fh.write("W_T_head " + " ".join(repr(float(x)) for x in W_T.reshape(-1)[:32]) + "\n")
    print(out)


if __name__ == "__main__":
    main()
