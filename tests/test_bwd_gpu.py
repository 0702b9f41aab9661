"""Parity of the scan's gradients (ssm_scan_bwd) with the backward oracle,
itself pinned by finite differences (needs a B200).

Tolerance: the kernel computes in fp32 (MUFU exponential and logarithm, sums
over up to a few hundred steps and over channels by atomics in any order);
every gradient must agree within 2e-3 of its largest magnitude."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import assert_close, dev
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu
GRAD_TOL = 2e-3


def _check(inp, dtype, softplus=True, use=("D", "z", "delta_bias", "h0"), seed=0):
    rng = np.random.default_rng(seed)
    dy = rng.standard_normal(inp["u"].shape).astype(np.float32)
    opt = lambda k, f: f(inp[k]) if k in use else None
    got = api.scan_bwd(dev(inp["u"], dtype), dev(inp["delta"], dtype), dev(inp["A"]),
                       dev(inp["B"], dtype), dev(inp["C"], dtype), dev(dy),
                       opt("D", dev), opt("z", lambda a: dev(a, dtype)), opt("delta_bias", dev),
                       softplus, opt("h0", dev))
    torch.cuda.synchronize()
    ref = oracle.scan_bwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], dy,
                          inp["D"] if "D" in use else None, inp["z"] if "z" in use else None,
                          inp["delta_bias"] if "delta_bias" in use else None, softplus,
                          inp["h0"] if "h0" in use else None)
    assert set(got) == set(ref), (sorted(got), sorted(ref))
    for k in ref:
        assert_close(got[k].cpu().numpy().astype(np.float64), ref[k], GRAD_TOL, k)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 17, 64, 300])
@pytest.mark.parametrize("dim,N", [(40, 16), (33, 5)])
def test_gradients_match_the_oracle(dtype, L, dim, N):
    inp = synth.make_scan_inputs(2, dim, N, L, dtype, gate=True, seed=L + dim, h0=True)
    _check(inp, dtype, seed=L)


@pytest.mark.parametrize("use", [(), ("D",), ("z",), ("delta_bias", "h0")])
def test_optional_inputs(use):
    inp = synth.make_scan_inputs(2, 48, 16, 100, "f32", gate=True, seed=3, h0=True)
    _check(inp, "f32", use=use, seed=1)


def test_without_softplus():
    inp = synth.make_scan_inputs(2, 32, 16, 80, "f32", gate=True, seed=4, h0=True)
    inp["delta"] = np.abs(inp["delta"]) * 0.05
    inp["delta_bias"] = np.full_like(inp["delta_bias"], 0.01)
    _check(inp, "f32", softplus=False, seed=2)
