"""Writes tests/golden/tiny_fp32_oracle.txt from the CPU oracle alone.

The pages print no worked numeric example, so this fixture is a regression
record of the oracle on the tiny fp32 workload (batch 1, 64 channels,
16 states, 256 steps, seed 0; inputs from the seeded generator).  It
catches unintended changes to the oracle's arithmetic; its correctness
rests on the pins, not on this file.  Run:  python tests/golden/make_golden.py
"""
import os
import sys

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.dirname(os.path.abspath(__file__))))
sys.path.insert(0, ROOT)

import oracle  # noqa: E402
from selective_state_space_08_b200 import synth  # noqa: E402

OUT = os.path.join(os.path.dirname(os.path.abspath(__file__)), "tiny_fp32_oracle.txt")
CHANNELS = (0, 17, 63)
STEPS = (0, 1, 2, 31, 100, 255)


def main():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                 cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"])
    y, h = oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], True, None, nthreads=1)
    with open(OUT, "w") as f:
        f.write("# oracle output, tiny fp32 workload (seed 0); written by make_golden.py\n")
        f.write("# kind channel index value\n")
        for d in CHANNELS:
            for t in STEPS:
                f.write(f"y {d} {t} {y[0, d, t]:.17e}\n")
            for n in range(cfg["dstate"]):
                f.write(f"h {d} {n} {h[0, d, n]:.17e}\n")
        f.write(f"ysum - - {float(np.sum(y)):.17e}\n")


if __name__ == "__main__":
    main()
