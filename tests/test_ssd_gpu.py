"""Parity of the chunked Mamba-2 (SSD) scan on the tensor cores with the CPU
oracle's sequential scalar-decay scan (needs a B200).  bf16 inputs:
max |y - y_ref| <= 2e-2 max |y_ref|, same bound on the final state."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _dev(a, bf=True):
    if a is None:
        return None
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).cuda()
    return t.to(torch.bfloat16) if bf else t


def _run(inp, chunk):
    y, h = api.ssd_fwd(_dev(inp["x"]), _dev(inp["delta"]), _dev(inp["A"], False), _dev(inp["B"]),
                       _dev(inp["C"]), _dev(inp["D"], False), _dev(inp["z"]),
                       _dev(inp["delta_bias"], False), True, _dev(inp["h0"], False), chunk=chunk,
                       check_status=True)
    return y.float().cpu().numpy(), h.cpu().numpy()


def _oracle(inp, heads=None):
    sel = slice(None) if heads is None else heads
    g = lambda k: None if inp[k] is None else inp[k]
    return oracle.ssd_fwd(inp["x"][:, :, sel], inp["delta"][:, :, sel], inp["A"][sel], inp["B"],
                          inp["C"], inp["D"][sel], None if g("z") is None else inp["z"][:, :, sel],
                          inp["delta_bias"][sel], True,
                          None if g("h0") is None else inp["h0"][:, sel])


@pytest.mark.parametrize("chunk", [128, 256])
@pytest.mark.parametrize("L,gate,h0", [(256, False, False), (300, True, True), (37, False, True),
                                       (1000, True, False), (512, False, True)])
def test_small_and_ragged(chunk, L, gate, h0):
    inp = synth.make_ssd_inputs(2, L, 3, 64, 128, "bf16", gate=gate, seed=L + chunk, h0=h0)
    y, h = _run(inp, chunk)
    yr, hr = _oracle(inp)
    assert_close(y, yr, TOL["bf16"], f"y L={L} chunk={chunk}")
    assert_close(h, hr, TOL["bf16"], f"h_L L={L} chunk={chunk}")


def test_chunk_lengths_agree():
    inp = synth.make_ssd_inputs(1, 768, 4, 64, 128, "bf16", gate=False, seed=77, h0=True)
    y1, h1 = _run(inp, 128)
    y2, h2 = _run(inp, 256)
    yr, hr = _oracle(inp)
    assert_close(y1, yr, TOL["bf16"], "chunk 128")
    assert_close(y2, yr, TOL["bf16"], "chunk 256")
    assert_close(h1, hr, TOL["bf16"], "chunk 128 h")
    assert_close(h2, hr, TOL["bf16"], "chunk 256 h")


def test_zero_length_keeps_h0():
    inp = synth.make_ssd_inputs(1, 0, 2, 64, 128, "bf16", gate=False, seed=5, h0=True)
    y, h = api.ssd_fwd(_dev(inp["x"]), _dev(inp["delta"]), _dev(inp["A"], False), _dev(inp["B"]),
                       _dev(inp["C"]), h0=_dev(inp["h0"], False), check_status=True)
    assert y.shape == (1, 0, 2, 64)
    assert np.array_equal(h.cpu().numpy(), inp["h0"])


@pytest.mark.slow
def test_mamba2_layer_sampled_heads():
    cfg = synth.CONFIGS["mamba2_ssd"]
    inp = synth.make_ssd_inputs(cfg["batch"], cfg["seqlen"], cfg["nheads"], cfg["headdim"],
                                cfg["dstate"], cfg["dtype"], cfg["gate"], cfg["seed"],
                                cfg["s_range"])
    y, h = _run(inp, cfg["chunk"])
    assert np.all(np.isfinite(y)) and np.all(np.isfinite(h))
    heads = [0, 17, 41, 79]
    yr, hr = _oracle(inp, heads)
    assert_close(y[:, :, heads], yr, TOL["bf16"], "mamba2 layer y (sampled heads)")
    assert_close(h[:, heads], hr, TOL["bf16"], "mamba2 layer h_L (sampled heads)")
