"""Mutation check of the oracle's pins (CPU only).

Each mutant is a copy of the C oracle with one plausible slip planted in it: a
dropped term, a flipped sign, a wrong or transposed index, an operand swapped.
The copy is compiled into a temporary directory and every pin is run against
it; the test requires at least one pin to reject it.  The oracle's own source
is never modified.  All mutants keep their memory accesses in bounds.
"""
import subprocess

import pytest

from oracle import oracle
from oracle_pins import PINS

# (name, exact snippet in ssm_oracle.c, replacement)
MUTANTS = [
    ("drop_D_term", "y += D[d] * x;", "y += 0.0 * x;"),
    ("exp_sign_flipped", "double a_bar = exp(dt * a_dn);", "double a_bar = exp(-dt * a_dn);"),
    ("B_read_from_C", "double b_tn = B[(b * dstate + n) * seqlen + t];",
     "double b_tn = C[(b * dstate + n) * seqlen + t];"),
    ("softplus_skipped", "if (softplus)\n                dt = oracle_softplus(dt);", ""),
    ("softplus_is_identity", "return log1p(exp(s));", "return log(exp(s));"),
    ("softplus_missing_one", "return log1p(exp(s));", "return log(exp(s) + 1e-3);"),
    ("bias_dropped", "dt += delta_bias[d];", "dt += 0.0;"),
    ("bias_after_softplus",
     "if (delta_bias)\n                dt += delta_bias[d];\n            if (softplus)\n"
     "                dt = oracle_softplus(dt);",
     "if (softplus)\n                dt = oracle_softplus(dt);\n            if (delta_bias)\n"
     "                dt += delta_bias[d];"),
    ("gate_sign_flipped", "return z / (1.0 + exp(-z));", "return z / (1.0 + exp(z));"),
    ("gate_is_sigmoid", "return z / (1.0 + exp(-z));", "return 1.0 / (1.0 + exp(-z));"),
    ("bbar_without_delta", "h[n] = a_bar * h[n] + gain * b_tn * x;",
     "h[n] = a_bar * h[n] + b_tn * x;"),
    ("state_not_decayed", "h[n] = a_bar * h[n] + gain * b_tn * x;",
     "h[n] = h[n] + gain * b_tn * x;"),
    ("readout_before_update",
     "h[n] = a_bar * h[n] + gain * b_tn * x;\n                y += c_tn * h[n];",
     "y += c_tn * h[n];\n                h[n] = a_bar * h[n] + gain * b_tn * x;"),
    ("B_time_shifted", "double b_tn = B[(b * dstate + n) * seqlen + t];",
     "double b_tn = B[(b * dstate + n) * seqlen + (t > 0 ? t - 1 : t)];"),
    ("C_batch_ignored", "double c_tn = C[(b * dstate + n) * seqlen + t];",
     "double c_tn = C[(0 * dstate + n) * seqlen + t];"),
    ("A_transposed", "double a_dn = A[d * dstate + n];\n                double a_bar",
     "double a_dn = A[n * dim + d];\n                double a_bar"),
    ("u_time_shifted", "double x = u_row[t];", "double x = u_row[t > 0 ? t - 1 : 0];"),
    ("last_state_zeroed", "last_state[(b * dim + d) * dstate + n] = h[n];",
     "last_state[(b * dim + d) * dstate + n] = 0.0 * h[n];"),
    ("update_state_not_decayed", "double h = a_bar * state[chain * dstate + n]",
     "double h = state[chain * dstate + n]"),
    ("update_bias_dropped", "delta += dt_bias[d];", "delta += 0.0;"),
    ("update_gate_dropped", "y *= oracle_silu(z[chain]);", "y *= 1.0;"),
    ("update_B_batch_ignored", "gain * B[b * dstate + n] * xv", "gain * B[n] * xv"),
    ("update_C_from_B", "y += C[b * dstate + n] * h;", "y += B[b * dstate + n] * h;"),
    ("update_D_dropped", "y += D[d] * xv;", "y += 0.0 * xv;"),
    ("update_softplus_skipped", "if (dt_softplus)\n            delta = oracle_softplus(delta);", ""),
    # zero-order hold and the start state
    ("zoh_gain_sign_flipped", "return expm1(dt * a) / a;", "return expm1(-dt * a) / a;"),
    ("zoh_gain_not_divided", "return expm1(dt * a) / a;", "return expm1(dt * a);"),
    ("zoh_gain_limit_dropped", "        return dt;\n    return expm1", "        return 0.0;\n    return expm1"),
    ("zoh_gain_uses_exp", "return expm1(dt * a) / a;", "return exp(dt * a) / a;"),
    ("zoh_ignored_in_scan", "double gain = zoh ? oracle_zoh_gain(dt, a_dn) : dt;",
     "double gain = dt;"),
    ("zoh_ignored_in_update", "double gain = zoh ? oracle_zoh_gain(delta, a_dn) : delta;",
     "double gain = delta;"),
    ("initial_state_ignored",
     "h[n] = initial_state ? initial_state[(b * dim + d) * dstate + n] : 0.0;", "h[n] = 0.0;"),
    ("initial_state_transposed", "initial_state[(b * dim + d) * dstate + n]",
     "initial_state[(d * batch + b) * dstate + n]"),
    # short causal convolution
    ("conv_tap_off_by_one", "int64_t s = t - (width - 1) + k;", "int64_t s = t - width + k;"),
    ("conv_state_index_shifted", "return state ? state[chain * width + (width + s)] : 0.0;",
     "return state ? state[chain * width + (width + s + 1) % width] : 0.0;"),
    ("conv_bias_dropped", "double acc = bias ? bias[d] : 0.0;\n            for",
     "double acc = 0.0;\n            for"),
    ("conv_silu_skipped", "out_row[t] = silu ? oracle_silu(acc) : acc;", "out_row[t] = acc;"),
    ("conv_weight_transposed", "acc += weight[d * width + k] *\n", "acc += weight[k * dim + d] *\n"),
    ("conv_final_state_reversed", "final_conv_state[chain * width + j] =",
     "final_conv_state[chain * width + (width - 1 - j)] ="),
    ("conv_update_not_shifted", "cur[j] = old[j + 1];", "cur[j] = old[j];"),
    ("conv_update_x_not_appended", "cur[width - 1] = x[chain];", "cur[width - 1] = old[width - 1];"),
    ("conv_update_bias_dropped", "double acc = bias ? bias[d] : 0.0;\n        for",
     "double acc = 0.0;\n        for"),
    # backward pass
    ("bwd_lambda_not_propagated", "lam[n] *= a_bar;", "lam[n] *= 1.0;"),
    ("bwd_dC_uses_previous_state", "+= dy * hs[(t + 1) * dstate + n];", "+= dy * hs[t * dstate + n];"),
    ("bwd_dA_missing_delta", "dA[d * dstate + n] += lam[n] * (dt * a_bar * h_prev",
     "dA[d * dstate + n] += lam[n] * (a_bar * h_prev"),
    ("bwd_softplus_grad_skipped", "double ds = softplus ? ddt * oracle_softplus_grad(s) : ddt;",
     "double ds = ddt;"),
    ("bwd_silu_grad_is_sigmoid", "return sg * (1.0 + z * (1.0 - sg));", "return sg;"),
    ("bwd_ddelta_A_term_sign", "ddt += lam[n] * (gain_dt * b_tn * x + a_dn * a_bar * h_prev);",
     "ddt += lam[n] * (gain_dt * b_tn * x - a_dn * a_bar * h_prev);"),
    ("bwd_du_missing_D", "double dut = D ? dy * D[d] : 0.0;", "double dut = 0.0;"),
    ("bwd_dB_missing_u", "+= lam[n] * gain * x;", "+= lam[n] * gain;"),
    # backward pass with the zero-order hold
    ("bwd_zoh_forward_is_euler", "double gain_f = zoh ? oracle_zoh_gain(dt, A[d * dstate + n]) : dt;",
     "double gain_f = dt;"),
    ("bwd_zoh_gain_is_euler", "double gain = zoh ? oracle_zoh_gain(dt, a_dn) : dt;\n                double gain_dt",
     "double gain = dt;\n                double gain_dt"),
    ("bwd_zoh_gain_dt_is_one", "double gain_dt = zoh ? a_bar : 1.0;", "double gain_dt = 1.0;"),
    ("bwd_zoh_gain_da_dropped", "double gain_da = zoh ? oracle_zoh_gain_da(dt, a_dn) : 0.0;",
     "double gain_da = 0.0;"),
    ("bwd_zoh_gain_da_sign", "return (x * exp(x) - expm1(x)) / (a * a);",
     "return (expm1(x) - x * exp(x)) / (a * a);"),
    ("bwd_zoh_gain_da_series_term", "(0.5 + x * (1.0 / 3.0 + x", "(0.5 + x * (1.0 / 2.0 + x"),
    ("bwd_zoh_du_uses_delta", "dut += lam[n] * gain * b_tn;", "dut += lam[n] * dt * b_tn;"),
    ("bwd_dlast_ignored", "lam[n] = dlast_state ? dlast_state[chain * dstate + n] : 0.0;",
     "lam[n] = 0.0;"),
    ("bwd_readout_grad_ungated", "dy = g * oracle_silu(zt);", "dy = g;"),
    ("bwd_dD_uses_dout", "dD[d] += dy * x;", "dD[d] += g * x;"),
    ("bwd_dh0_one_step_late", "dinitial_state[chain * dstate + n] = lam[n];",
     "dinitial_state[chain * dstate + n] = lam[n] * exp(dts[0] * A[d * dstate + n]);"),
    # Mamba-2 layer (scalar A per head)
    ("ssd_group_interleaved", "int64_t g = h / heads_per_group;", "int64_t g = h % ngroups;"),
    ("ssd_decay_sign_flipped", "double decay = exp(delta * A[h]);",
     "double decay = exp(-delta * A[h]);"),
    ("ssd_input_without_delta", "S_p[n] = decay * S_p[n] + delta * x_t[p] * B_t[n];",
     "S_p[n] = decay * S_p[n] + x_t[p] * B_t[n];"),
    ("ssd_readout_before_update",
     "S_p[n] = decay * S_p[n] + delta * x_t[p] * B_t[n];\n                    y += C_t[n] * S_p[n];",
     "y += C_t[n] * S_p[n];\n                    S_p[n] = decay * S_p[n] + delta * x_t[p] * B_t[n];"),
    ("ssd_C_read_from_B", "y += C_t[n] * S_p[n];", "y += B_t[n] * S_p[n];"),
    ("ssd_D_dropped", "y += D[h] * x_t[p];", "y += 0.0 * x_t[p];"),
    ("ssd_gate_dropped", "y *= oracle_silu(z_t[p]);", "y *= 1.0;"),
    ("ssd_bias_dropped", "delta += dt_bias[h];", "delta += 0.0;"),
    ("ssd_softplus_skipped", "if (dt_softplus)\n                delta = oracle_softplus(delta);", ""),
    ("ssd_initial_state_ignored",
     "S[i] = initial_state ? initial_state[chain * headdim * dstate + i] : 0.0;", "S[i] = 0.0;"),
    ("ssd_final_state_stale", "final_state[chain * headdim * dstate + i] = S[i];",
     "final_state[chain * headdim * dstate + i] = initial_state ? initial_state[chain * headdim * dstate + i] : 0.0;"),
    ("ssd_headdim_reversed", "y += D[h] * x_t[p];", "y += D[h] * x_t[headdim - 1 - p];"),
    ("ssd_dt_time_shifted", "double delta = dt[(b * seqlen + t) * nheads + h];",
     "double delta = dt[(b * seqlen + (t > 0 ? t - 1 : 0)) * nheads + h];"),
]


def test_mutant_snippets_present():
    src = oracle.SOURCE.read_text()
    for name, old, _ in MUTANTS:
        assert old in src, f"mutant {name}: snippet not found in the oracle source"


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = oracle.SOURCE.read_text()
    assert old in src
    mutated = tmp_path / f"{name}.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = tmp_path / f"lib{name}.so"
    try:
        oracle.build(mutated, lib, force=True)
    except subprocess.CalledProcessError as e:  # pragma: no cover - a mutant must compile
        pytest.fail(f"mutant {name} does not compile: {e}")
    handle = oracle.Oracle(lib)
    caught = []
    for pin_name, pin in PINS.items():
        try:
            pin(handle)
        except AssertionError:
            caught.append(pin_name)
    assert caught, f"mutant {name} passed every pin"
