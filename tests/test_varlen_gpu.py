"""Parity of the packed variable-length scan (ssm_scan_fwd_varlen) with the
CPU oracle run sequence by sequence (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close, dev
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _pack(lengths, dim, dtype, seed):
    inp = synth.make_scan_inputs(1, dim, 16, int(sum(lengths)), dtype, gate=True, seed=seed)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return inp, cu


def _oracle(inp, cu):
    ys, hs = [], []
    for i in range(len(cu) - 1):
        sl = slice(int(cu[i]), int(cu[i + 1]))
        y, h = oracle.scan_fwd(inp["u"][..., sl], inp["delta"][..., sl], inp["A"],
                               inp["B"][..., sl], inp["C"][..., sl], inp["D"], inp["z"][..., sl],
                               inp["delta_bias"], True, None)
        ys.append(y)
        hs.append(h[0])
    return np.concatenate(ys, axis=-1), np.stack(hs)


def _run(inp, cu, dtype):
    y, h = api.scan_fwd_varlen(dev(inp["u"], dtype), dev(inp["delta"], dtype), dev(inp["A"]),
                               dev(inp["B"], dtype), dev(inp["C"], dtype),
                               torch.from_numpy(cu).cuda(), dev(inp["D"]), dev(inp["z"], dtype),
                               dev(inp["delta_bias"]), True)
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), h.cpu().numpy()


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("lengths", [[1, 63, 64, 65, 130, 7, 300], [2048], [5] * 50,
                                     [64] * 6, [1] * 20 + [500]])
def test_packed_sequences_match_separate_scans(dtype, lengths):
    inp, cu = _pack(lengths, 70, dtype, seed=len(lengths) + sum(lengths))
    y, h = _run(inp, cu, dtype)
    yr, hr = _oracle(inp, cu)
    assert_close(y, yr, TOL[dtype], f"y {lengths[:4]}")
    assert_close(h, hr, TOL[dtype], f"h_L {lengths[:4]}")


def test_packed_sequences_across_segments():
    """Few channels and a long packed row: the scan runs in L-segments, with
    restarts inside segments cutting the carried state."""
    rng = np.random.default_rng(3)
    lengths = list(rng.integers(1, 900, size=20))
    inp, cu = _pack(lengths, 32, "bf16", seed=44)
    y, h = _run(inp, cu, "bf16")
    yr, hr = _oracle(inp, cu)
    assert_close(y, yr, TOL["bf16"], "y")
    assert_close(h, hr, TOL["bf16"], "h_L")
