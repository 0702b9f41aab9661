"""Parity of the CUDA selective scan with the CPU oracle (needs a B200).

Small and ragged shapes are compared element by element; the full-size
workloads (the launch configurations the benchmark times) are compared on
sampled channels, which the oracle computes over the whole sequence."""
import numpy as np
import pytest
import torch

import oracle
from gpu_util import TOL, assert_close, dev, inputs_for, run_scan
from selective_state_space_08_b200 import api, synth

pytestmark = pytest.mark.gpu


def _oracle(inp, softplus=True, use_h0=True, use_D=True, use_bias=True, use_z=True):
    return oracle.scan_fwd(inp["u"], inp["delta"], inp["A"], inp["B"], inp["C"],
                           inp["D"] if use_D else None, inp["z"] if use_z else None,
                           inp["delta_bias"] if use_bias else None, softplus,
                           inp["h0"] if use_h0 else None)


def test_tiny_fp32_every_element():
    cfg, inp = inputs_for("tiny_fp32")
    y, h = run_scan(inp, "f32")
    yr, hr = _oracle(inp)
    assert_close(y, yr, TOL["f32"], "y")
    assert_close(h, hr, TOL["f32"], "h_L")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("L", [1, 7, 64, 255, 1000, 4097])
@pytest.mark.parametrize("dim,N", [(1, 16), (45, 5), (33, 1), (64, 16)])
def test_ragged_shapes(dtype, L, dim, N):
    inp = synth.make_scan_inputs(2, dim, N, L, dtype, gate=True, seed=L * 7 + dim, h0=True)
    y, h = run_scan(inp, dtype)
    yr, hr = _oracle(inp)
    assert_close(y, yr, TOL[dtype], f"y L={L} dim={dim} N={N}")
    assert_close(h, hr, TOL[dtype], f"h_L L={L} dim={dim} N={N}")


@pytest.mark.parametrize("opts", [
    dict(softplus=False), dict(use_h0=False), dict(use_D=False), dict(use_bias=False),
    dict(use_z=False), dict(use_z=False, use_D=False, use_bias=False, use_h0=False)])
@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_optional_inputs(dtype, opts):
    inp = synth.make_scan_inputs(3, 70, 16, 300, dtype, gate=True, seed=5, h0=True)
    if opts.get("softplus") is False:  # keep dt' = delta + bias positive and moderate
        inp["delta"] = np.abs(inp["delta"]) * 0.05
        inp["delta_bias"] = np.full_like(inp["delta_bias"], 0.01)
    y, h = run_scan(inp, dtype, **opts)
    yr, hr = _oracle(inp, **opts)
    assert_close(y, yr, TOL[dtype], f"y {opts}")
    assert_close(h, hr, TOL[dtype], f"h_L {opts}")


def test_strided_views_and_scalar_path():
    """Sliced (non-contiguous) inputs and rows that break 16-byte alignment."""
    inp = synth.make_scan_inputs(2, 40, 16, 203, "bf16", gate=True, seed=9, h0=True)
    wide = {k: (np.concatenate([v, v[..., :13]], axis=-1) if k in ("u", "delta", "z", "B", "C")
                else v) for k, v in inp.items()}
    t = {k: (dev(v, "bf16") if k in ("u", "delta", "z", "B", "C") else dev(v))
         for k, v in wide.items()}
    L = 203
    y, h = api.scan_fwd(t["u"][..., :L], t["delta"][..., :L], t["A"], t["B"][..., :L],
                        t["C"][..., :L], t["D"], t["z"][..., :L], t["delta_bias"], True, t["h0"])
    yr, hr = _oracle(inp)
    assert_close(y.float().cpu().numpy(), yr, TOL["bf16"], "strided y")
    assert_close(h.cpu().numpy(), hr, TOL["bf16"], "strided h_L")


def test_segmented_sequence_and_split_resume():
    """Few channels and a long sequence: the L-segment path, then the same scan
    split at m = L/2 and resumed from h_m through strided halves."""
    L, dim = 1 << 16, 40
    inp = synth.make_scan_inputs(1, dim, 16, L, "bf16", gate=True, seed=31, s_range=(1e-4, 1e-2),
                                 h0=True)
    args = [dev(inp["u"], "bf16"), dev(inp["delta"], "bf16"), dev(inp["A"]),
            dev(inp["B"], "bf16"), dev(inp["C"], "bf16"), dev(inp["D"]), dev(inp["z"], "bf16"),
            dev(inp["delta_bias"])]
    assert api.scan_fwd_workspace_size(*args[:5]) > 0  # the sequence is split
    y, h = api.scan_fwd(*args, True, dev(inp["h0"]))
    yr, hr = _oracle(inp)
    assert_close(y.float().cpu().numpy(), yr, TOL["bf16"], "segmented y")
    assert_close(h.cpu().numpy(), hr, TOL["bf16"], "segmented h_L")
    m = L // 2
    u, dl, A, B, C, D, z, bias = args
    y1, hm = api.scan_fwd(u[..., :m], dl[..., :m], A, B[..., :m], C[..., :m], D, z[..., :m], bias,
                          True, dev(inp["h0"]))
    y2, h2 = api.scan_fwd(u[..., m:], dl[..., m:], A, B[..., m:], C[..., m:], D, z[..., m:], bias,
                          True, hm)
    ys = torch.cat([y1, y2], dim=-1).float().cpu().numpy()
    assert_close(ys, yr, TOL["bf16"], "split-resume y")
    assert_close(h2.cpu().numpy(), hr, TOL["bf16"], "split-resume h_L")


def test_zero_length_and_empty_batch():
    A = torch.full((4, 16), -1.0, device="cuda")
    h0 = torch.randn(2, 4, 16, device="cuda")
    e = torch.empty(2, 4, 0, device="cuda")
    bc = torch.empty(2, 16, 0, device="cuda")
    y, h = api.scan_fwd(e, e, A, bc, bc, h0=h0)
    torch.cuda.synchronize()
    assert y.shape == (2, 4, 0) and torch.equal(h, h0)
    y, h = api.scan_fwd(e, e, A, bc, bc)
    torch.cuda.synchronize()
    assert torch.count_nonzero(h) == 0
    z0 = torch.empty(0, 4, 5, device="cuda")
    y, h = api.scan_fwd(z0, z0, A, torch.empty(0, 16, 5, device="cuda"),
                        torch.empty(0, 16, 5, device="cuda"))
    assert y.shape == (0, 4, 5)


def _sampled(name, batches, dims, **over):
    """The full-size workload on the GPU; the oracle on sampled channels."""
    cfg = dict(synth.CONFIGS[name])
    cfg.update(over)
    full = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                  cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"], bits=True)
    y, h = api.scan_fwd(dev(full["u"]), dev(full["delta"]), dev(full["A"]), dev(full["B"]),
                        dev(full["C"]), dev(full["D"]), dev(full["z"]), dev(full["delta_bias"]),
                        True, None)
    torch.cuda.synchronize()
    assert bool(torch.isfinite(y.float()).all()) and bool(torch.isfinite(h).all())
    del full
    worst = 0.0
    for b in batches:
        chans = [(b, d) for d in dims]
        s = synth.make_scan_inputs(cfg["batch"], cfg["dim"], cfg["dstate"], cfg["seqlen"],
                                   cfg["dtype"], cfg["gate"], cfg["seed"], cfg["s_range"],
                                   channels=chans)
        yr, hr = oracle.scan_fwd(s["u"], s["delta"], s["A"], s["B"], s["C"], s["D"], s["z"],
                                 s["delta_bias"], True, None)
        idx = torch.tensor(dims, device="cuda")
        yg = y[b].index_select(0, idx).float().cpu().numpy()[None]
        hg = h[b].index_select(0, idx).cpu().numpy()[None]
        worst = max(worst, assert_close(yg, yr, TOL[cfg["dtype"]], f"{name} y b={b}"))
        assert_close(hg, hr, TOL[cfg["dtype"]], f"{name} h_L b={b}")
    return worst


@pytest.mark.slow
def test_mamba130m_layer_sampled():
    _sampled("mamba130m_layer", [0, 7], [0, 1, 31, 32, 33, 700, 1535])


@pytest.mark.slow
@pytest.mark.parametrize("gate", [True, False])
def test_mamba2p8b_layer_sampled(gate):
    _sampled("mamba2p8b_layer", [0, 3], [0, 63, 2500, 5119], gate=gate)


@pytest.mark.slow
def test_long_sequence_sampled():
    _sampled("long_seq", [0], [0, 517, 1023])


def test_decode_steps_match_the_sequence_scan_and_the_oracle():
    inp = synth.make_scan_inputs(3, 50, 16, 24, "f32", gate=True, seed=41, h0=True)
    y_seq, h_seq = run_scan(inp, "f32")
    st = dev(inp["h0"]).clone()
    A, D, bias = dev(inp["A"]), dev(inp["D"]), dev(inp["delta_bias"])
    ys = []
    st_o = inp["h0"].astype(np.float64)
    for t in range(24):
        args = [dev(np.ascontiguousarray(inp[k][..., t])) for k in ("u", "delta")]
        Bt, Ct = dev(np.ascontiguousarray(inp["B"][..., t])), dev(np.ascontiguousarray(inp["C"][..., t]))
        zt = dev(np.ascontiguousarray(inp["z"][..., t]))
        ys.append(api.scan_step(st, args[0], args[1], A, Bt, Ct, D, zt, bias, True))
        yo, st_o = oracle.scan_step(st_o, inp["u"][..., t], inp["delta"][..., t], inp["A"],
                                    inp["B"][..., t], inp["C"][..., t], inp["D"], inp["z"][..., t],
                                    inp["delta_bias"], True)
        assert_close(ys[-1].cpu().numpy(), yo, TOL["f32"], f"step y t={t}")
    torch.cuda.synchronize()
    assert_close(torch.stack(ys, -1).cpu().numpy(), y_seq, TOL["f32"], "steps vs scan y")
    assert_close(st.cpu().numpy(), h_seq, TOL["f32"], "steps vs scan state")


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("N", [16, 7])
def test_decode_step_bf16_and_ragged_states(dtype, N):
    inp = synth.make_scan_inputs(4, 37, N, 1, dtype, gate=True, seed=43, h0=True)
    st = dev(inp["h0"]).clone()
    y = api.scan_step(st, dev(np.ascontiguousarray(inp["u"][..., 0]), dtype),
                      dev(np.ascontiguousarray(inp["delta"][..., 0]), dtype), dev(inp["A"]),
                      dev(np.ascontiguousarray(inp["B"][..., 0]), dtype),
                      dev(np.ascontiguousarray(inp["C"][..., 0]), dtype), dev(inp["D"]),
                      dev(np.ascontiguousarray(inp["z"][..., 0]), dtype), dev(inp["delta_bias"]))
    yo, so = oracle.scan_step(inp["h0"], inp["u"][..., 0], inp["delta"][..., 0], inp["A"],
                              inp["B"][..., 0], inp["C"][..., 0], inp["D"], inp["z"][..., 0],
                              inp["delta_bias"])
    torch.cuda.synchronize()
    assert_close(y.float().cpu().numpy(), yo, TOL[dtype], "step y")
    assert_close(st.cpu().numpy(), so, TOL[dtype], "step state")
