"""Writes tests/golden/tiny_sweep.txt from the oracle alone (regression fixture).

Run: python tests/golden/make_golden.py
The fixture holds the oracle's codes for the seeded tiny layer (W [64,128]
fp32, X [256,128] bf16); it pins later oracle edits to the reviewed result.
"""
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(os.path.dirname(HERE)))

import numpy as np  # noqa: E402

import oracle  # noqa: E402
import synth  # noqa: E402


def main():
    L = synth.make_config(0)
    W = L.W_f32()[0]
    A = oracle.absmax(W)
    H = oracle.hessian(L.X)
    codes, amax, err = oracle.sweep(W, [A], H)
    with open(os.path.join(HERE, "tiny_sweep.txt"), "w") as f:
        f.write("# oracle codes for synth.make_config(0) (tiny layer), rows of 8 block columns\n")
        f.write(f"global_amax {float(A).hex()}\n")
        f.write(f"sum_err {float(err.sum()).hex()}\n")
        for r in range(codes.shape[1]):
            f.write(" ".join(str(int(c)) for c in codes[0, r]) + "\n")


if __name__ == "__main__":
    main()
