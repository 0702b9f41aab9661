"""Parity of the scan with grouped B and C (ngroups > 1) with the CPU oracle
run group by group (needs a B200)."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close, dev
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _inputs(batch, dim, L, G, dtype, seed):
    inp = synth.make_scan_inputs(batch, dim, 16, L, dtype, gate=True, seed=seed, h0=True)
    inp.update(synth.make_grouped_bc(batch, G, 16, L, dtype, seed=seed))
    return inp


def _oracle(inp, G):
    dim = inp["u"].shape[1]
    cpg = dim // G
    ys, hs = [], []
    for g in range(G):
        sl = slice(g * cpg, (g + 1) * cpg)
        y, h = oracle.scan_fwd(inp["u"][:, sl], inp["delta"][:, sl], inp["A"][sl], inp["B"][:, g],
                               inp["C"][:, g], inp["D"][sl], inp["z"][:, sl],
                               inp["delta_bias"][sl], True, inp["h0"][:, sl])
        ys.append(y)
        hs.append(h)
    return np.concatenate(ys, axis=1), np.concatenate(hs, axis=1)


def _args(inp, dtype):
    return (dev(inp["u"], dtype), dev(inp["delta"], dtype), dev(inp["A"]), dev(inp["B"], dtype),
            dev(inp["C"], dtype), dev(inp["D"]), dev(inp["z"], dtype), dev(inp["delta_bias"]),
            True, dev(inp["h0"]))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("G,dim", [(2, 64), (4, 128), (3, 192)])
@pytest.mark.parametrize("L", [7, 300])
def test_grouped_matches_oracle_per_group(dtype, G, dim, L):
    inp = _inputs(2, dim, L, G, dtype, seed=G * 100 + L)
    y, h = api.scan_fwd(*_args(inp, dtype))
    torch.cuda.synchronize()
    yr, hr = _oracle(inp, G)
    assert_close(y.float().cpu().numpy(), yr, TOL[dtype], f"y G={G}")
    assert_close(h.cpu().numpy(), hr, TOL[dtype], f"h_L G={G}")


def test_grouped_segmented_and_strided():
    """Few channels and a long sequence (L-segments), with B and C taken as
    views of larger tensors (non-default group and batch strides)."""
    G, dim, L = 2, 64, 6000
    inp = _inputs(1, dim, L, G, "bf16", seed=77)
    a = list(_args(inp, "bf16"))
    big = torch.zeros((1, G + 1, 16, L + 64), dtype=torch.bfloat16, device="cuda")
    big[:, 1:, :, :L] = a[3]
    a[3] = big[:, 1:, :, :L]                 # group stride 16*(L+64), state stride L+64
    y, h = api.scan_fwd(*a)
    torch.cuda.synchronize()
    yr, hr = _oracle(inp, G)
    assert_close(y.float().cpu().numpy(), yr, TOL["bf16"], "y")
    assert_close(h.cpu().numpy(), hr, TOL["bf16"], "h_L")


def test_grouped_from_host_buffers():
    G, dim, L = 4, 128, 200
    inp = _inputs(3, dim, L, G, "f32", seed=5)
    host = lambda k: torch.from_numpy(np.ascontiguousarray(inp[k], dtype=np.float32)).pin_memory()
    y, h = api.scan_fwd_host(host("u"), host("delta"), host("A"), host("B"), host("C"), host("D"),
                             host("z"), host("delta_bias"), True, host("h0"), slice_batch=2)
    yr, hr = _oracle(inp, G)
    assert_close(y.numpy(), yr, TOL["f32"], "y")
    assert_close(h.numpy(), hr, TOL["f32"], "h_L")
