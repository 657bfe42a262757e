"""The oracle's pins catch plausible mistakes.

Each case plants one mistake in a temporary copy of oracle/s6_oracle.c (on the
CPU, never in the CUDA path), builds it, routes the oracle through it, and
checks that at least one pin of test_oracle_pins.py now fails.
"""
import os
import subprocess

import pytest

from oracle import s6_oracle as O
import test_oracle_block as TK
import test_oracle_bwd as TB
import test_oracle_diag as TD
import test_oracle_pins as P

SRC = os.path.join(os.path.dirname(O.__file__), "s6_oracle.c")

ALL_PINS = [
    P.test_recorded_decays_exact,
    P.test_recorded_decays_in_unit_interval,
    P.test_recorded_first_state_equals_first_write,
    P.test_recorded_update_rule_exact,
    P.test_recorded_changed_token_carries_through_decay_only,
    P.test_state_sizes,
    lambda: [P.test_softplus_against_libm(v) for v in (-7.0, -1e-3, 0.5, 21.0)],
    P.test_softplus_zero_is_ln2,
    lambda: [P.test_silu_against_libm(v) for v in (-10.0, 0.7, 5.0)],
    P.test_A_is_negative_exp,
    P.test_zoh_gain_tends_to_delta,
    P.test_geometric_series_simplified,
    P.test_zoh_matches_continuous_time_solution,
    lambda: P.test_bruteforce_decayed_sum(False),
    lambda: P.test_bruteforce_decayed_sum(True),
    P.test_readout_uses_updated_state,
    P.test_conv_onehot_taps_shift,
    P.test_conv_against_numpy_convolve,
    P.test_D_multiplies_conv_output_and_gate,
    P.test_future_changes_leave_past_unchanged,
    P.test_conv_window_width3,
    lambda: P.test_streaming_equals_full_forward(True),
    TB.test_sigmoid_and_dsilu_closed_forms,
    lambda: TB.check_gradients_by_central_differences(False, True),
    lambda: TB.check_gradients_by_central_differences(True, True),
    lambda: TB.check_fused_gradients_by_central_differences(False),
    TD.test_diag_bruteforce_decayed_sum,
    TD.test_diag_geometric_series,
    TD.test_diag_equals_selective_scan_at_unit_step,
    TD.test_diag_decays_in_unit_interval_and_state_bounded,
    TD.test_diag_streaming_continues_from_state,
    TK.test_block_worked_example,
    TK.test_block_streaming_equals_sequence_form,
    TK.test_linear_q8_against_numpy,
    TK.test_layernorm_against_numpy,
]

MUTATIONS = {
    "decay_sign": ("return exp(delta * s6o_A(A_log));", "return exp(-delta * s6o_A(A_log));"),
    "A_not_exp": ("double s6o_A(double A_log) { return -exp(A_log); }",
                  "double s6o_A(double A_log) { return -A_log; }"),
    "update_minus": ("return a_bar * h + write;", "return a_bar * h - write;"),
    "update_no_decay": ("return a_bar * h + write;", "return h + write;"),
    "zoh_missing_minus_one": ("return expm1(delta * A) / A;", "return exp(delta * A) / A;"),
    "zoh_missing_div_A": ("return expm1(delta * A) / A;", "return -expm1(delta * A);"),
    "zoh_as_simplified": ("    if (!zoh)\n        return delta;", "    if (zoh >= 0)\n        return delta;"),
    "readout_old_state": ("            h[n] = s6o_update(h[n], a_bar, write);\n            acc += h[n] * Cm[t * N + n];",
                          "            acc += h[n] * Cm[t * N + n];\n            h[n] = s6o_update(h[n], a_bar, write);"),
    "C_index_transposed": ("acc += h[n] * Cm[t * N + n];", "acc += h[n] * Cm[n * N + t % N];"),
    "B_is_C": ("* Bm[t * N + n] * u;", "* Cm[t * N + n] * u;"),
    "D_on_preconv": ("double out = acc + D * u;", "double out = acc + D * x[t];"),
    "no_gate_silu": ("out *= s6o_silu(z[t]);", "out *= z[t];"),
    "no_dt_bias": ("s6o_softplus(dt_raw[t] + dt_bias);", "s6o_softplus(dt_raw[t]);"),
    "softplus_drop_max": ("return m + log1p(exp(-fabs(v)));", "return log1p(exp(-fabs(v)));"),
    "silu_is_sigmoid": ("return v / (1.0 + exp(-v));", "return 1.0 / (1.0 + exp(-v));"),
    "conv_taps_reversed": ("acc += w[k] * hist[k];", "acc += w[K - 2 - k] * hist[k];"),
    "conv_no_bias": ("double acc = bias;", "double acc = 0.0 * bias;"),
    "conv_history_not_shifted": ("hist[k] = hist[k + 1];", "hist[k] = hist[k];"),
    "state_count_wrong": ("return d_inner * d_state * blocks;", "return d_inner * d_state;"),
    # the backward pass
    "bwd_carry_no_decay": ("g[n] = dh * a_bar;   /* to h_{t-1} */", "g[n] = dh;   /* to h_{t-1} */"),
    "bwd_zoh_explicit_dA_missing": ("dA += dgain * (delta * a_bar * A - expm1(delta * A)) / (A * A);",
                                    "dA += 0.0 * dgain;"),
    "bwd_no_softplus_derivative": ("double dv = ddelta * s6o_sigmoid(v);", "double dv = ddelta;"),
    "bwd_dA_log_chain_missing": ("dA_log[n] += dA * A;", "dA_log[n] += dA;"),
    "bwd_dsilu_as_sigmoid": ("return s * (1.0 + v * (1.0 - s));", "return s;"),
    "bwd_dC_old_state": ("dC[t * N + n] += ds * h_t[n];", "dC[t * N + n] += ds * h_prev[n];"),
    "bwd_du_misses_D": ("double dut = ds * D;", "double dut = 0.0 * ds;"),
    "bwd_gate_not_applied": ("double ds = dy[t] * gate;", "double ds = dy[t];"),
    "bwd_write_gain_missing_in_dB": ("dB[t * N + n] += dh * gain * u[t];", "dB[t * N + n] += dh * u[t];"),
    "cbwd_no_dsilu": ("double dpre = dxc[c * L + t] * s6o_dsilu(pre);", "double dpre = dxc[c * L + t];"),
    "cbwd_dx_taps_reversed": ("dxo[src] += w[k] * dpre;", "dxo[src] += w[K - 1 - k] * dpre;"),
    "cbwd_dw_wrong_input": ("dw[c * K + k] += dpre * xc[src];", "dw[c * K + k] += dpre * xc[t];"),
    # the constant-decay cell
    "diag_decay_sign": ("a[n] = exp2(log2_decay[n]);", "a[n] = exp2(-log2_decay[n]);"),
    "diag_decay_natural_base": ("a[n] = exp2(log2_decay[n]);", "a[n] = exp(log2_decay[n]);"),
    "diag_write_without_u": ("Bm[t * N + n] * u[t]);", "Bm[t * N + n]);"),
    "diag_readout_old_state": ("            h[n] = s6o_update(h[n], a[n], Bm[t * N + n] * u[t]);\n            acc += h[n] * Cm[t * N + n];",
                               "            acc += h[n] * Cm[t * N + n];\n            h[n] = s6o_update(h[n], a[n], Bm[t * N + n] * u[t]);"),
    "diag_no_skip": ("double out = acc + D * u[t];", "double out = acc;"),
    "diag_B_is_C": ("h[n] = s6o_update(h[n], a[n], Bm[t * N + n] * u[t]);", "h[n] = s6o_update(h[n], a[n], Cm[t * N + n] * u[t]);"),
    # the decode block
    "block_no_residual": ("        x[i] += o[i];", "        x[i] = o[i];"),
    "block_ln_unbiased_variance": ("    var /= n;", "    var /= (n - 1);"),
    "block_ln_no_affine_bias": ("out[i] = (x[i] - mean) * r * w[i] + b[i];", "out[i] = (x[i] - mean) * r * w[i];"),
    "block_linear_scale_per_column": ("y[o] = scale[o] * acc;", "y[o] = scale[o % n_in] * acc;"),
    "block_xproj_B_C_swapped": ("const double *Bt = dbc + R, *Ct = dbc + R + N;", "const double *Bt = dbc + R + N, *Ct = dbc + R;"),
    "block_dt_bias_missing": ("double delta = s6o_softplus(dtr[c] + p->dt_bias[c]);", "double delta = s6o_softplus(dtr[c]);"),
    "block_gate_from_xin": ("g[c] = yv * s6o_silu(xz[di + c]);", "g[c] = yv * s6o_silu(xz[c]);"),
    "block_conv_history_not_updated": ("            hist[K - 2] = xz[c];", "            hist[K - 2] = hist[K - 2];"),
}


def _build_mutant(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, name
    src = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib_{name}.so"
    c.write_text(src)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    return str(so)


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    so = _build_mutant(tmp_path, name)
    failed = []
    with O.use_library(so):
        for pin in ALL_PINS:
            try:
                pin()
            except AssertionError:
                failed.append(pin)
    assert failed, f"no pin caught mutation {name}"


def test_unmutated_copy_passes_all(tmp_path):
    c = tmp_path / "same.c"
    so = tmp_path / "lib_same.so"
    c.write_text(open(SRC).read())
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", str(so), str(c), "-lm"])
    with O.use_library(str(so)):
        for pin in ALL_PINS:
            pin()
