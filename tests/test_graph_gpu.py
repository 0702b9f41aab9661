"""The library's calls captured in a CUDA graph (needs a B200).

They allocate nothing and never synchronise, so a sequence of them can be
captured once and replayed, which removes the per-call launch latency that
dominates a decode step or a short sequence.  Replays must give exactly the
results of the same calls made one by one, and the oracle's."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close, dev
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _capture(fn):
    """fn() once on a side stream (one-time setup such as the shared-memory
    opt-in happens outside the graph), then captured into a graph."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        fn()
    torch.cuda.current_stream().wait_stream(side)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    return g


def test_decode_steps_replayed_from_a_graph():
    T, batch, dim = 16, 4, 96
    inp = synth.make_scan_inputs(batch, dim, 16, T, "bf16", gate=True, seed=21, h0=True)
    col = lambda k, t: dev(np.ascontiguousarray(inp[k][..., t]), "bf16")
    steps = [dict(u=col("u", t), delta=col("delta", t), B=col("B", t), C=col("C", t),
                  z=col("z", t)) for t in range(T)]
    A, D, bias = dev(inp["A"]), dev(inp["D"]), dev(inp["delta_bias"])
    h0 = dev(inp["h0"])

    def run(state, ys):
        for t, s in enumerate(steps):
            api.scan_step(state, s["u"], s["delta"], A, s["B"], s["C"], D, s["z"], bias, True,
                          y=ys[t])

    y_eager = [torch.empty((batch, dim), dtype=torch.bfloat16, device="cuda") for _ in range(T)]
    st_eager = h0.clone()
    run(st_eager, y_eager)
    y_graph = [torch.empty_like(y) for y in y_eager]
    st_graph = h0.clone()
    g = _capture(lambda: run(st_graph, y_graph))
    st_graph.copy_(h0)  # the capture's warm-up advanced the state
    g.replay()
    torch.cuda.synchronize()
    for t in range(T):
        assert torch.equal(y_graph[t], y_eager[t]), f"step {t}"
    assert torch.equal(st_graph, st_eager)
    yr, hr = oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                             inp["z"], inp["delta_bias"], True, inp["h0"])
    yg = torch.stack(y_graph, dim=-1).float().cpu().numpy()
    assert_close(yg, yr, TOL["bf16"], "y")
    assert_close(st_graph.cpu().numpy(), hr, TOL["bf16"], "state")


def test_segmented_scan_replayed_from_a_graph():
    """The 1 x 64 x 16 x 256 fp32 case runs as three launches (aggregate pass,
    carry fold, full pass); replayed from a graph it matches the eager call."""
    inp = synth.make_scan_inputs(1, 64, 16, 256, "f32", gate=True, seed=0, h0=True)
    t = {k: dev(v) for k, v in inp.items() if v is not None}
    args = (t["u"], t["delta"], t["A"], t["B"], t["C"], t["D"], t["z"], t["delta_bias"], True,
            t["h0"])
    need = api.scan_fwd_workspace_size(*args)
    assert need > 0, "expected the segmented path"
    ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    y_eager, h_eager = api.scan_fwd(*args, workspace=ws)
    y_graph, h_graph = torch.empty_like(y_eager), torch.empty_like(h_eager)
    g = _capture(lambda: api.scan_fwd(*args, y=y_graph, h_last=h_graph, workspace=ws))
    y_graph.zero_()
    h_graph.zero_()
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(y_graph, y_eager) and torch.equal(h_graph, h_eager)
    yr, hr = oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"], inp["D"],
                             inp["z"], inp["delta_bias"], True, inp["h0"])
    assert_close(y_graph.cpu().numpy(), yr, TOL["f32"], "y")
