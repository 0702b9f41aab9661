"""Helpers for the GPU parity tests: upload seeded inputs, run the library
through its binding, compare with the oracle under the stated tolerances."""
from __future__ import annotations

import numpy as np
import torch

from selective_state_space_08_b200 import api, synth

# max |got - ref| <= TOL[dtype] * max |ref|   (fp32 inputs: 1e-4; bf16 inputs: 2e-2)
TOL = {"f32": 1e-4, "bf16": 2e-2}
TORCH = {"f32": torch.float32, "bf16": torch.bfloat16}


def dev(x, dtype="f32"):
    """numpy -> CUDA tensor: float32 values (exactly representable in dtype)
    or uint16 bfloat16 bit patterns."""
    if x is None:
        return None
    if x.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(x).view(np.int16)).cuda().view(torch.bfloat16)
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    return t.to(TORCH[dtype]) if dtype != "f32" else t


def run_scan(inp, dtype, softplus=True, use_h0=True, use_D=True, use_bias=True, use_z=True):
    y, h = api.scan_fwd(dev(inp["u"], dtype), dev(inp["delta"], dtype), dev(inp["A"]),
                        dev(inp["B"], dtype), dev(inp["C"], dtype),
                        dev(inp["D"]) if use_D else None,
                        dev(inp["z"], dtype) if use_z else None,
                        dev(inp["delta_bias"]) if use_bias else None, softplus,
                        dev(inp["h0"]) if use_h0 else None)
    torch.cuda.synchronize()
    return y.float().cpu().numpy().astype(np.float64), h.cpu().numpy().astype(np.float64)


def max_rel_err(got, ref):
    got = np.asarray(got, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    if ref.size == 0:
        return 0.0
    scale = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (scale if scale > 0 else 1.0)


def assert_close(got, ref, tol, what):
    assert got.shape == ref.shape, (what, got.shape, ref.shape)
    assert np.all(np.isfinite(got)), f"{what}: non-finite output"
    err = max_rel_err(got, ref)
    assert err <= tol, f"{what}: max|err| / max|ref| = {err:.3e} > {tol:.1e}"
    return err


def inputs_for(name, **over):
    cfg = dict(synth.CONFIGS[name])
    cfg.update(over)
    return cfg, synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                       cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"])
