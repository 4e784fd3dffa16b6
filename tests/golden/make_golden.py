"""Write the oracle regression fixtures: linear_tiny_f32_seed0.txt,
mlp_small_seed0.txt and linear_decode_pieces_seed0.txt.

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


MLP_KEYS = ("Q", "K", "V", "eta", "W1_0", "b1_0", "W2_0", "b2_0", "gamma", "beta")
DECODE_CUTS = (5, 6, 21, 33)


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

    # TTT-MLP: the 8k workload's recipe at B=1, H=1, T=48
    w = WORKLOADS["mlp_8k"].with_shape(B=1, H=1, T=48)
    inp = make_inputs(w, 0)
    Z, W1_T, b1_T, W2_T, b2_T = oracle.ttt_mlp(*(inp[k] for k in MLP_KEYS), w.mini_batch, w.ln_eps)
    idx = np.random.default_rng(4321).choice(Z.size, 48, replace=False)
    idx.sort()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "mlp_small_seed0.txt")
    with open(out, "w") as fh:
        fh.write("# Oracle regression values: TTT-MLP, B=1 H=1 T=48 d=64 hidden=256 b=16, bf16 inputs,\n")
        fh.write("# seed 0 (mlp_8k recipe).  Written by make_golden.py from the float64 oracle only.\n")
        fh.write("Z_index " + " ".join(str(int(i)) for i in idx) + "\n")
        fh.write("Z " + " ".join(repr(float(x)) for x in Z.reshape(-1)[idx]) + "\n")
        fh.write("W2_T_head " + " ".join(repr(float(x)) for x in W2_T.reshape(-1)[:32]) + "\n")
        fh.write("b1_T_head " + " ".join(repr(float(x)) for x in b1_T.reshape(-1)[:16]) + "\n")
    print(out)

    # TTT-Linear decode in pieces (125M recipe at B=1, H=1, T=40; b = 16)
    w = WORKLOADS["linear_125m_2k"].with_shape(B=1, H=1, T=40)
    inp = make_inputs(w, 0)
    W, b, W_mb, b_mb = inp["W0"], inp["b0"], None, None
    Zs = []
    bounds = [0, *DECODE_CUTS, w.T]
    for a, c in zip(bounds[:-1], bounds[1:]):
        sl = lambda x: x[:, :, a:c]
        Zp, W, b, W_mb, b_mb = oracle.ttt_linear_decode(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["eta"]),
                                                        W, b, W_mb, b_mb, inp["gamma"], inp["beta"], 16, a % 16)
        Zs.append(Zp)
    Z = np.concatenate(Zs, axis=2)
    idx = np.random.default_rng(2468).choice(Z.size, 48, replace=False)
    idx.sort()
    out = os.path.join(os.path.dirname(os.path.abspath(__file__)), "linear_decode_pieces_seed0.txt")
    with open(out, "w") as fh:
        fh.write("# Oracle regression values: TTT-Linear decode, B=1 H=1 T=40 d=64 b=16, bf16 inputs, seed 0\n")
        fh.write("# (125M recipe), decoded in pieces cut at DECODE_CUTS.  Written by make_golden.py from the\n")
        fh.write("# float64 oracle only.\n")
        fh.write("cuts " + " ".join(str(c) for c in DECODE_CUTS) + "\n")
        fh.write("Z_index " + " ".join(str(int(i)) for i in idx) + "\n")
        fh.write("Z " + " ".join(repr(float(x)) for x in Z.reshape(-1)[idx]) + "\n")
        fh.write("W_mb_head " + " ".join(repr(float(x)) for x in W_mb.reshape(-1)[:32]) + "\n")
    print(out)


if __name__ == "__main__":
    main()
