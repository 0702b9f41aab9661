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
    # step size: the bias must act with softplus off too, and the cutoff
    # where softplus(s) is taken as s must sit where the two agree
    ("softplus_off_drops_bias", "return softplus ? softplus_d(s) : s;",
     "return softplus ? softplus_d(s) : delta;", ALL_PINS),
    ("softplus_cutoff_too_low", "return s > 20.0 ? s : log1p(exp(s)); }",
     "return s > 2.0 ? s : log1p(exp(s)); }", ALL_PINS),
    # the selective scan: batch and time indexing of the shared and per-row terms
    ("B_from_batch_0", "const double* Bb = j->B + b * N * L;", "const double* Bb = j->B;",
     MAMBA1_PINS),
    ("h0_ignores_batch", "h[n] = j->h0 ? j->h0[row * N + n] : 0.0;",
     "h[n] = j->h0 ? j->h0[d * N + n] : 0.0;", MAMBA1_PINS),
    ("skip_uses_previous_u", "(j->D ? j->D[d] * u[t] : 0.0)",
     "(j->D ? j->D[d] * u[t > 0 ? t - 1 : 0] : 0.0)", MAMBA1_PINS),
    ("gate_time_shift", "if (j->z) yv *= silu_d(j->z[row * L + t]);",
     "if (j->z) yv *= silu_d(j->z[row * L + (t > 0 ? t - 1 : 0)]);", MAMBA1_PINS),
    # the decode step
    ("step_drop_skip", "double yv = acc + (D ? D[d] * u[row] : 0.0);", "double yv = acc;",
     MAMBA1_PINS),
    ("step_drop_gate", "if (z) yv *= silu_d(z[row]);", "if (0) yv *= silu_d(z[row]);",
     MAMBA1_PINS),
    ("step_ignores_bias", "step_size(delta[row], bias, d, softplus)",
     "step_size(delta[row], NULL, d, softplus)", MAMBA1_PINS),
    # the scalar-decay scan
    ("ssd_drop_gate", "if (j->z) yv *= silu_d(j->z[xo + p]);",
     "if (0) yv *= silu_d(j->z[xo + p]);", SSD_PINS),
    ("ssd_ignores_bias", "step_size(j->delta[(b * L + t) * H + hd], j->bias, hd, j->softplus)",
     "step_size(j->delta[(b * L + t) * H + hd], NULL, hd, j->softplus)", SSD_PINS),
    ("ssd_B_time_shift", "const double* Bt = j->B + (b * L + t) * N;",
     "const double* Bt = j->B + (b * L + (t > 0 ? t - 1 : 0)) * N;", SSD_PINS),
    ("ssd_x_of_head_0", "const int64_t xo = ((b * L + t) * H + hd) * P;",
     "const int64_t xo = ((b * L + t) * H) * P;", SSD_PINS),
    # gradients
    ("bwd_dC_uses_h_prev", "if (dC) dC[b * N * L + n * L + t] += ds * hs[(t + 1) * N + n];",
     "if (dC) dC[b * N * L + n * L + t] += ds * hs[t * N + n];", BWD_PINS),
    ("bwd_dD_ungated", "dDd += ds * ur[t];", "dDd += dy[row * L + t] * ur[t];", BWD_PINS),
    ("bwd_dB_no_dt", "if (dB) dB[b * N * L + n * L + t] += lam[n] * dt * ur[t];",
     "if (dB) dB[b * N * L + n * L + t] += lam[n] * ur[t];", BWD_PINS),
    ("bwd_ddelta_skips_softplus", "const double dd = softplus ? ddt * softplus_grad(sarg) : ddt;",
     "const double dd = ddt;", BWD_PINS),
    ("bwd_dz_without_skip", "double sv = D ? D[d] * ur[t] : 0.0;", "double sv = 0.0;", BWD_PINS),
    ("bwd_adjoint_without_readout", "lam[n] += ds * Cb[n * L + t];", "lam[n] += 0.0 * ds;",
     BWD_PINS),
    ("ssd_C_time_shift", "const double* Ct = j->C + (b * L + t) * N;",
     "const double* Ct = j->C + (b * L + (t > 0 ? t - 1 : 0)) * N;", SSD_PINS),
    ("ssd_h_last_zero", "j->h_last[row * P * N + i] = S[i];", "j->h_last[row * P * N + i] = 0.0;",
     SSD_PINS),
    ("conv_first_tap_only", "for (int64_t k = 0; k < K; ++k) {", "for (int64_t k = 0; k < 1; ++k) {",
     CONV_PINS),
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
