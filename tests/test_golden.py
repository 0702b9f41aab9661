"""The oracle against its stored record on the tiny fp32 workload (no GPU)."""
import os

import numpy as np

import oracle
from selective_state_space_08_b200 import synth

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "tiny_fp32_oracle.txt")


def test_oracle_matches_golden_record():
    cfg = synth.CONFIGS["tiny_fp32"]
    inp = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                 cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"])
    y, h = oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                           inp["z"], inp["delta_bias"], True, None, nthreads=3)
    n = 0
    for line in open(GOLDEN):
        if line.startswith("#"):
            continue
        kind, a, b, v = line.split()
        v = float(v)
        if kind == "y":
            got = y[0, int(a), int(b)]
        elif kind == "h":
            got = h[0, int(a), int(b)]
        else:
            got = float(np.sum(y))
        assert abs(got - v) <= 1e-12 * max(1.0, abs(v)), (kind, a, b, got, v)
        n += 1
    assert n > 50
