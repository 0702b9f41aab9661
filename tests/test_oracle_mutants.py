"""Planted mistakes in the oracle must each be caught by at least one pin.

Every mutant is a textual edit of a copy of ``oracle/ssm_oracle.c``,
compiled into a temporary directory and run on the CPU against the pins.
A pin that can no longer see a dropped term, a flipped sign, a swapped
operand or a shifted index would let such a mistake through unnoticed.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS, BWD_PINS, CONV_PINS, MAMBA1_PINS, SSD_PINS

SRC = os.path.join(os.path.dirname(oracle.__file__), "ssm_oracle.c")

# (name, original text, replacement, which pins must catch it)
MUTANTS = [
    ("drop_skip", "(j->D ? j->D[d] * u[t] : 0.0)", "0.0", MAMBA1_PINS),
    ("gate_sign", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));", ALL_PINS),
    ("decay_sign", "const double dA = exp(dt * Ad[n]);", "const double dA = exp(-dt * Ad[n]);",
     MAMBA1_PINS),
    ("input_no_dt", "dt * Bb[n * L + t] * u[t]", "Bb[n * L + t] * u[t]", MAMBA1_PINS),
    ("readout_uses_B", "acc += Cb[n * L + t] * h[n];", "acc += Bb[n * L + t] * h[n];", MAMBA1_PINS),
    ("readout_before_update",
     "h[n] = dA * h[n] + dBu;                       /* h_t = A_d h_{t-1} + B_d u_t */\n"
     "        acc += Cb[n * L + t] * h[n];",
     "acc += Cb[n * L + t] * h[n];\n        h[n] = dA * h[n] + dBu;", MAMBA1_PINS),
    ("softplus_is_exp", "s > 20.0 ? s : log1p(exp(s))", "s > 20.0 ? s : exp(s)", ALL_PINS),
    ("bias_outside_softplus",
     "double s = delta + (bias ? bias[d] : 0.0);\n  return softplus ? softplus_d(s) : s;",
     "return (softplus ? softplus_d(delta) : delta) + (bias ? bias[d] : 0.0);", ALL_PINS),
    ("ignore_h0", "h[n] = j->h0 ? j->h0[row * N + n] : 0.0;", "h[n] = 0.0;", MAMBA1_PINS),
    ("B_time_shift", "const double dBu = dt * Bb[n * L + t] * u[t];",
     "const double dBu = dt * Bb[n * L + (t > 0 ? t - 1 : 0)] * u[t];", MAMBA1_PINS),
    ("A_transposed", "const double* Ad = j->A + d * N;", "const double* Ad = j->A + (d % N) * N;",
     MAMBA1_PINS),
    ("h_last_zero", "j->h_last[row * N + n] = h[n];", "j->h_last[row * N + n] = 0.0;", MAMBA1_PINS),
    ("step_wrong_A_row", "exp(dt * A[d * dstate + n])", "exp(dt * A[n])", MAMBA1_PINS),
    ("ssd_head0_decay", "const double a = exp(dt * j->A[hd]);", "const double a = exp(dt * j->A[0]);",
     SSD_PINS),
    ("ssd_input_no_dt", "dt * xv * Bt[n]", "xv * Bt[n]", SSD_PINS),
    ("ssd_readout_uses_B", "acc += Ct[n] * S[p * N + n];", "acc += Bt[n] * S[p * N + n];", SSD_PINS),
    ("ssd_drop_skip", "(j->D ? j->D[hd] * xv : 0.0)", "0.0", SSD_PINS),
    ("ssd_ignore_h0", "S[i] = j->h0 ? j->h0[row * P * N + i] : 0.0;", "S[i] = 0.0;", SSD_PINS),
    ("conv_taps_reversed", "acc += j->w[d * K + k] * xv;", "acc += j->w[d * K + (K - 1 - k)] * xv;",
     CONV_PINS),
    ("conv_no_bias", "double acc = j->bias ? j->bias[d] : 0.0;", "double acc = 0.0;", CONV_PINS),
    ("conv_no_silu", "j->u[row * L + t] = silu_d(acc);", "j->u[row * L + t] = acc;", CONV_PINS),
    ("conv_ignores_window", "else if (j->x_prev)", "else if (0)", CONV_PINS),
    ("conv_time_shift", "const int64_t tt = t - (K - 1) + k;", "const int64_t tt = t - K + k;",
     CONV_PINS),
    ("bwd_adjoint_not_decayed", "lam[n] *= a;                                      /* carried",
     "lam[n] *= 1.0;                                    /* carried", BWD_PINS),
    ("bwd_du_no_dt", "du_t += lam[n] * dt * Bb[n * L + t];", "du_t += lam[n] * Bb[n * L + t];",
     BWD_PINS),
    ("bwd_dA_uses_h_t", "if (dA) dA[d * N + n] += lam[n] * dt * a * hp;",
     "if (dA) dA[d * N + n] += lam[n] * dt * a * hs[(t + 1) * N + n];", BWD_PINS),
    ("bwd_softplus_grad", "return s > 20.0 ? 1.0 : 1.0 / (1.0 + exp(-s));",
     "return s > 20.0 ? 1.0 : 1.0 / (1.0 + exp(s));", BWD_PINS),
    ("bwd_gate_grad", "(sg * (1.0 + zv * (1.0 - sg)))", "(sg * (1.0 + zv * sg))", BWD_PINS),
]


def _fails(pin, lib):
    try:
        pin(lib)
    except (AssertionError, FloatingPointError, ValueError, RuntimeError):
        return True
    return False


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc not available")
@pytest.mark.parametrize("name,old,new,pins", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new, pins):
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site of {name} not found exactly once"
    mpath = tmp_path / "mutant.c"
    mpath.write_text(src.replace(old, new))
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-O2", "-fPIC", "-shared", "-std=c11", "-o", so, str(mpath), "-lm",
                    "-lpthread"], check=True)
    lib = oracle.load(so)
    caught = [p.__name__ for p in pins if _fails(p, lib)]
    assert caught, f"mutant {name} passes every pin"
