"""The seeded input generator: sampled channels regenerate exactly the rows of
a full draw (what the full-size parity tests rely on to run the oracle on a
few channels), draws are deterministic, bf16 values are exact, and the
distributions follow the stated recipe."""
import numpy as np
import pytest

from selective_state_space_08_b200 import synth


def test_sampled_channels_equal_the_rows_of_a_full_draw():
    batch, dim, N, L = 2, 130, 16, 100   # channels span three 64-row generator blocks
    full = synth.make_scan_inputs(batch, dim, N, L, "bf16", gate=True, seed=5, h0=True)
    chans = [(1, 0), (1, 63), (1, 64), (1, 127), (1, 129)]
    part = synth.make_scan_inputs(batch, dim, N, L, "bf16", gate=True, seed=5, h0=True,
                                  channels=chans)
    ds = [d for _, d in chans]
    for k in ("u", "delta", "z", "h0"):
        np.testing.assert_array_equal(part[k][0], full[k][1][ds], err_msg=k)
    for k in ("A", "D", "delta_bias"):
        np.testing.assert_array_equal(part[k], full[k][ds], err_msg=k)
    for k in ("B", "C"):
        np.testing.assert_array_equal(part[k][0], full[k][1], err_msg=k)


def test_sampled_channels_must_share_a_batch():
    with pytest.raises(ValueError):
        synth.make_scan_inputs(2, 8, 4, 10, channels=[(0, 1), (1, 1)])


def test_draws_are_seeded_and_deterministic():
    a = synth.make_scan_inputs(1, 8, 4, 32, "f32", seed=3)
    b = synth.make_scan_inputs(1, 8, 4, 32, "f32", seed=3)
    c = synth.make_scan_inputs(1, 8, 4, 32, "f32", seed=4)
    for k in ("u", "delta", "z", "B", "C", "A", "D", "delta_bias"):
        np.testing.assert_array_equal(a[k], b[k], err_msg=k)
        assert not np.array_equal(a[k], c[k]), k


def test_bf16_values_are_exact_and_bits_match():
    f = synth.make_scan_inputs(1, 16, 4, 64, "bf16", seed=1)
    bits = synth.make_scan_inputs(1, 16, 4, 64, "bf16", seed=1, bits=True)
    for k in ("u", "delta", "z", "B", "C"):
        assert bits[k].dtype == np.uint16
        np.testing.assert_array_equal(synth.bf16_bits_to_f32(bits[k]), f[k], err_msg=k)
        np.testing.assert_array_equal(synth.to_bf16_bits(f[k]), bits[k], err_msg=k)


def test_distributions_follow_the_recipe():
    dim, N = 4096, 16
    inp = synth.make_scan_inputs(1, dim, N, 64, "f32", seed=11, s_range=(1e-3, 1e-1))
    # A = -exp(U(ln 1, ln 10))
    assert inp["A"].max() <= -1.0 and inp["A"].min() >= -10.0
    la = np.log(-inp["A"].astype(np.float64))
    assert abs(la.mean() - np.log(10) / 2) < 5 * np.log(10) / np.sqrt(12 * dim * N)
    # softplus(bias) log-uniform in [1e-3, 1e-1]
    s = np.log1p(np.exp(inp["delta_bias"].astype(np.float64)))
    assert s.min() >= 1e-3 * (1 - 1e-5) and s.max() <= 1e-1 * (1 + 1e-5)
    width = np.log(1e-1) - np.log(1e-3)   # uniform in log space: sd = width / sqrt(12)
    assert abs(np.log(s).mean() - (np.log(1e-3) + np.log(1e-1)) / 2) < 5 * width / np.sqrt(12 * dim)
    # the sequence tensors and D are standard normal: mean and standard
    # deviation within 5 standard errors of 0 and 1
    for k in ("u", "delta", "z", "B", "C", "D"):
        v = inp[k].astype(np.float64).ravel()
        n = v.size
        assert abs(v.mean()) < 5 / np.sqrt(n), k
        assert abs(v.std() - 1.0) < 5 * np.sqrt(0.5 / n), k
