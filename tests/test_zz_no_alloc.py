"""ssm_scan_fwd_noalloc: the selective scan for callers that cannot allocate
device memory (a host framework that owns all device buffers and forbids
allocation while it runs, or a latency-critical path that cannot take
cudaMalloc's implicit synchronisation).  Its scratch is the library's static
device array instead of a caller-provided workspace; its results must match
ssm_scan_fwd's.  Collected last so that a stop at the first failure has
already run every other test."""
import ctypes

import numpy as np
import pytest
import torch

from gpu_util import TOL, dev
from selective_state_space_08_b200 import _abi, api, synth

pytestmark = pytest.mark.gpu


def _case(seed):
    # one batch, 64 channels, 2^16 steps: few channels, so the sequence is split
    # into segments and the scan needs scratch for the segment carries
    inp = synth.make_scan_inputs(1, 64, 16, 1 << 16, "bf16", gate=True, seed=seed,
                                 s_range=(1e-4, 1e-2), h0=True)
    return [dev(inp["u"], "bf16"), dev(inp["delta"], "bf16"), dev(inp["A"]),
            dev(inp["B"], "bf16"), dev(inp["C"], "bf16"), dev(inp["D"]), dev(inp["z"], "bf16"),
            dev(inp["delta_bias"]), True, dev(inp["h0"])]


def test_noalloc_matches_scan_fwd_on_two_calls_in_a_row():
    lib = _abi.load()
    for seed in (101, 202):
        args = _case(seed)
        need = api.scan_fwd_workspace_size(*args)
        assert 0 < need <= 4 << 20  # uses scratch, and fits the static array
        y_ref, h_ref = api.scan_fwd(*args)
        y = torch.empty_like(y_ref)
        h = torch.empty_like(h_ref)
        a = api._scan_args(*args, y, h)
        stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
        _abi.check(lib.ssm_scan_fwd_noalloc(ctypes.byref(a), stream), "ssm_scan_fwd_noalloc")
        torch.cuda.synchronize()
        for got, ref, what in ((y, y_ref, "y"), (h, h_ref, "h_L")):
            g = got.float().cpu().numpy()
            r = ref.float().cpu().numpy()
            assert np.all(np.isfinite(g)), what
            err = float(np.max(np.abs(g - r)) / np.max(np.abs(r)))
            assert err <= TOL["bf16"], (seed, what, err)
