"""Writes tests/golden/tiny_oracle.txt from the float64 oracle alone.

The pages print no numeric VDA value, so this fixture is not a pin: it is a
regression anchor for the oracle on the tiny workload (B=1, H=1, T=8, n=64,
d=64, 16 text tokens, FP32, lam=1, seed 0), whose values are fixed by the
oracle as pinned in tests/test_oracle_pins.py.  Run from the repository root:
    python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

from frame_wise_linear_b200 import synth  # noqa: E402
from oracle import vda_oracle as vo  # noqa: E402

SAMPLES = 48


def compute():
    inp = synth.make_inputs("tiny", seed=0)
    w = inp.workload
    f = lambda k: inp.widened(k)  # noqa: E731
    O, states = vo.vda_forward(f("Q"), f("K"), f("V"), f("G"), f("K_txt"), f("V_txt"), w.lam, return_states=True)
    rng = np.random.default_rng(12345)
    idx = [tuple(int(rng.integers(0, s)) for s in O.shape) for _ in range(SAMPLES)]
    return O, states[0], idx


def main():
    O, st, idx = compute()
    path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_oracle.txt")
    with open(path, "w") as fh:
        fh.write("# VDA forward, tiny workload, seed 0; written by tests/golden/make_golden.py from oracle/ only.\n")
        fh.write("# Regression anchor for the oracle (the pages print no numeric value for VDA).\n")
        fh.write(f"frob_O {np.linalg.norm(O):.17g}\n")
        for t in range(st["SF"].shape[0]):
            fh.write(f"frob_SF {t} {np.linalg.norm(st['SF'][t]):.17g}\n")
            fh.write(f"frob_SB {t} {np.linalg.norm(st['SB'][t]):.17g}\n")
        for i in idx:
            fh.write("O " + " ".join(str(x) for x in i) + f" {O[i]:.17g}\n")


if __name__ == "__main__":
    main()
