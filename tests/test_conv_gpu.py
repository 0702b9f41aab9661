"""Parity of the scan with the fused convolution stage (ssm_scan_fwd_conv)
with the CPU oracle (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close, dev
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _run(inp, conv, dtype, use_bias=True, use_prev=True, h0=True, x=None):
    x = inp["u"] if x is None else x
    y, h = api.scan_fwd_conv(dev(x, dtype), dev(conv["weight"]),
                             dev(conv["bias"]) if use_bias else None,
                             dev(conv["x_prev"]) if (use_prev and conv["x_prev"] is not None)
                             else None,
                             dev(inp["delta"], dtype), dev(inp["A"]), dev(inp["B"], dtype),
                             dev(inp["C"], dtype), dev(inp["D"]), dev(inp["z"], dtype),
                             dev(inp["delta_bias"]), True, dev(inp["h0"]) if h0 else None)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64), h.cpu().numpy().astype(np.float64)


def _oracle(inp, conv, use_bias=True, use_prev=True, h0=True, x=None):
    x = inp["u"] if x is None else x
    return oracle.scan_fwd_conv(x, conv["weight"], conv["bias"] if use_bias else None,
                                conv["x_prev"] if use_prev else None, inp["delta"], inp["A"],
                                inp["B"], inp["C"], inp["D"], inp["z"], inp["delta_bias"], True,
                                inp["h0"] if h0 else None)


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("width", [1, 2, 3, 4])
@pytest.mark.parametrize("L", [1, 5, 64, 130, 1000])
def test_widths_and_ragged_lengths(dtype, width, L):
    inp = synth.make_scan_inputs(2, 45, 16, L, dtype, gate=True, seed=L + 3 * width, h0=True)
    conv = synth.make_conv_params(45, width, seed=width, batch=2, prev=True)
    y, h = _run(inp, conv, dtype)
    yr, hr = _oracle(inp, conv)
    assert_close(y, yr, TOL[dtype], f"y width={width} L={L}")
    assert_close(h, hr, TOL[dtype], f"h_L width={width} L={L}")


@pytest.mark.parametrize("opts", [dict(use_bias=False), dict(use_prev=False),
                                  dict(use_bias=False, use_prev=False, h0=False)])
def test_optional_parameters(opts):
    inp = synth.make_scan_inputs(3, 70, 16, 300, "bf16", gate=True, seed=5, h0=True)
    conv = synth.make_conv_params(70, 4, seed=2, batch=3, prev=True)
    y, h = _run(inp, conv, "bf16", **opts)
    yr, hr = _oracle(inp, conv, **opts)
    assert_close(y, yr, TOL["bf16"], f"y {opts}")
    assert_close(h, hr, TOL["bf16"], f"h_L {opts}")


def test_segmented_sequence():
    """Few channels and a long sequence: the scan runs in L-segments, each
    segment's convolution window reaching back into the previous one."""
    inp = synth.make_scan_inputs(1, 40, 16, 9000, "bf16", gate=True, seed=8, h0=True)
    conv = synth.make_conv_params(40, 4, seed=3, batch=1, prev=True)
    y, h = _run(inp, conv, "bf16")
    yr, hr = _oracle(inp, conv)
    assert_close(y, yr, TOL["bf16"], "y")
    assert_close(h, hr, TOL["bf16"], "h_L")


def test_split_and_resume():
    """[0, m) then [m, L) with x_prev = the last three inputs before m and
    h0 = the first call's h_last equals one call."""
    inp = synth.make_scan_inputs(2, 33, 16, 400, "f32", gate=True, seed=12, h0=True)
    conv = synth.make_conv_params(33, 4, seed=4, batch=2, prev=True)
    yr, hr = _oracle(inp, conv)
    m = 137
    first = {k: (v[..., :m] if k in ("u", "delta", "z", "B", "C") else v) for k, v in inp.items()}
    y1, h1 = _run(first, conv, "f32")
    second = {k: (np.ascontiguousarray(v[..., m:]) if k in ("u", "delta", "z", "B", "C") else v)
              for k, v in inp.items()}
    second["h0"] = h1.astype(np.float32)
    conv2 = dict(conv, x_prev=np.ascontiguousarray(inp["u"][..., m - 3:m]))
    y2, h2 = _run(second, conv2, "f32")
    assert_close(np.concatenate([y1, y2], axis=-1), yr, TOL["f32"], "y split")
    assert_close(h2, hr, TOL["f32"], "h_L split")


@pytest.mark.slow
def test_mamba130m_layer_sampled():
    """The full-size 130M-layer workload with the stage in front, against
    the oracle on sampled channels."""
    cfg = synth.CONFIGS["mamba130m_layer"]
    full = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                  cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"], bits=True)
    conv = synth.make_conv_params(cfg["dim"], 4, seed=1)
    y, h = api.scan_fwd_conv(dev(full["u"]), dev(conv["weight"]), dev(conv["bias"]), None,
                             dev(full["delta"]), dev(full["A"]), dev(full["B"]), dev(full["C"]),
                             dev(full["D"]), dev(full["z"]), dev(full["delta_bias"]), True, None)
    torch.cuda.synchronize()
    del full
    dims = [0, 1, 700, 1535]
    for b in (0, 7):
        s = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                   cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"],
                                   channels=[(b, d) for d in dims])
        yr, hr = oracle.scan_fwd_conv(s["u"], conv["weight"][dims], conv["bias"][dims], None,
                                      s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"],
                                      s["delta_bias"], True, None)
        idx = torch.tensor(dims, device="cuda")
        assert_close(y[b].index_select(0, idx).float().cpu().numpy()[None], yr, TOL["bf16"],
                     f"y b={b}")
        assert_close(h[b].index_select(0, idx).cpu().numpy()[None], hr, TOL["bf16"], f"h_L b={b}")
