"""Parity of the host-resident scan (ssm_scan_fwd_host: batch slices
pipelined through device staging) with the CPU oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _cpu(x, dtype, pin):
    """numpy -> CPU tensor (float32 values, or uint16 bfloat16 bit patterns)."""
    if x is None:
        return None
    if x.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
        if dtype == "bf16" and x.ndim == 3:
            t = t.to(torch.bfloat16)
    t = t.contiguous()
    return t.pin_memory() if pin else t


def _run(inp, dtype, slice_batch, pin=True, use_h0=True, use_z=True, use_D=True, use_bias=True,
         last_state=True):
    f = lambda k, on=True: _cpu(inp[k], dtype, pin) if on else None
    y, h = api.scan_fwd_host(f("u"), f("delta"), _cpu(inp["A"], "f32", pin), f("B"), f("C"),
                             _cpu(inp["D"], "f32", pin) if use_D else None, f("z", use_z),
                             _cpu(inp["delta_bias"], "f32", pin) if use_bias else None, True,
                             _cpu(inp["h0"], "f32", pin) if use_h0 else None,
                             slice_batch=slice_batch, return_last_state=last_state)
    y = y.float().numpy().astype(np.float64)
    return y, (None if h is None else h.numpy().astype(np.float64))


def _oracle(inp, use_h0=True, use_z=True, use_D=True, use_bias=True):
    return oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                           inp["D"] if use_D else None, inp["z"] if use_z else None,
                           inp["delta_bias"] if use_bias else None, True,
                           inp["h0"] if use_h0 else None)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("slice_batch", [1, 2, 5, 9])
def test_slices_match_oracle(dtype, slice_batch):
    """Batch 5 in slices of 1, 2 (ragged last slice), 5 and 9 (one slice)."""
    inp = synth.make_scan_inputs(5, 70, 16, 333, dtype, gate=True, seed=11 + slice_batch, h0=True)
    y, h = _run(inp, dtype, slice_batch)
    yr, hr = _oracle(inp)
    assert_close(y, yr, TOL[dtype], f"y slice_batch={slice_batch}")
    assert_close(h, hr, TOL[dtype], f"h_L slice_batch={slice_batch}")


def test_optional_inputs_and_pageable_memory():
    inp = synth.make_scan_inputs(3, 40, 7, 150, "bf16", gate=True, seed=3, h0=True)
    opts = dict(use_h0=False, use_z=False, use_D=False, use_bias=False)
    y, h = _run(inp, "bf16", 2, pin=False, **opts)
    yr, hr = _oracle(inp, **opts)
    assert_close(y, yr, TOL["bf16"], "y")
    assert_close(h, hr, TOL["bf16"], "h_L")


def test_without_last_state_and_long_slices():
    """A slice whose scan runs in L-segments (few channels, long sequence)."""
    inp = synth.make_scan_inputs(2, 32, 16, 5000, "bf16", gate=True, seed=4, h0=True)
    y, h = _run(inp, "bf16", 1, last_state=False)
    assert h is None
    yr, _ = _oracle(inp)
    assert_close(y, yr, TOL["bf16"], "y")


def test_zero_length_passes_the_state_through():
    inp = synth.make_scan_inputs(3, 20, 16, 0, "f32", gate=True, seed=2, h0=True)
    y, h = _run(inp, "f32", 2)
    assert y.shape == (3, 20, 0)
    assert np.array_equal(h, inp["h0"].astype(np.float64))


@pytest.mark.slow
def test_bench_workload_sampled():
    """The end-to-end benchmark's call (130M layer from page-locked host
    memory, slices of one sequence): sampled channels against the oracle."""
    cfg = synth.CONFIGS["mamba130m_layer"]
    full = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                  cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"], bits=True)
    y, h = _run(full, cfg["dtype"], 1, use_h0=False)
    del full
    dims = [0, 1, 777, 1535]
    for b in (0, 7):
        s = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                   cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"],
                                   channels=[(b, d) for d in dims])
        yr, hr = oracle.scan_fwd(s["u"], s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"],
                                 s["delta_bias"], True, None)
        assert_close(y[b, dims][None], yr, TOL["bf16"], f"y b={b}")
        assert_close(h[b, dims][None], hr, TOL["bf16"], f"h_L b={b}")
