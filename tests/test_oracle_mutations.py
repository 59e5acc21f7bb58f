"""The oracle's pins catch plausible mistakes.

Each case plants one slip in a temporary copy of the oracle's C source (on the
CPU, never on a GPU), rebuilds it, and reruns the pins of
``test_oracle_pins.py``, ``test_oracle_bwd_pins.py`` and
``test_oracle_mamba3_pins.py`` against the mutant: at least one pin must fail.
"""
import importlib.util
import os
import sys

import pytest

import tests.test_oracle_bwd_pins as bwd_pins
import tests.test_oracle_mamba3_pins as m3_pins
import tests.test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "ssd_oracle.c")

# (name, original text, mutated text); every original must occur in the source
MUTATIONS = [
    ("y_before_state_update",   # recurrence: read the state before the token-t update
     "            /* h_t = decay * h_{t-1} + dt * B_t x_t^T */\n",
     "            if (y) { double* yt0 = y + ((b * L + t) * H + h) * P; for (int64_t p = 0; p < P; ++p) { double a0 = 0.0; for (int64_t n = 0; n < N; ++n) a0 += Ct[n] * st[n * P + p]; yt0[p] = a0 + d_skip * xt[p]; } }\n            if (0)\n"),
    ("decay_sign", "const double decay = exp(dt * A[h]);\n            const double* xt = x + ((b * L + t)",
     "const double decay = exp(-dt * A[h]);\n            const double* xt = x + ((b * L + t)"),
    ("b_c_swapped_in_recurrence", "const double coef = dt * Bt[n];", "const double coef = dt * Ct[n];"),
    ("skip_term_dropped", "yt[p] = acc + d_skip * xt[p];", "yt[p] = acc;"),
    ("group_map_modulo", "for (pair = 0; pair < batch * H; ++pair) {\n        const int64_t b = pair / H, h = pair % H, g = h / heads_per_group;\n        double* st",
     "for (pair = 0; pair < batch * H; ++pair) {\n        const int64_t b = pair / H, h = pair % H, g = h % G;\n        double* st"),
    ("euler_dt_missing", "const double coef = dt * Bt[n];", "const double coef = Bt[n];"),
    ("quadratic_exclusive_cumsum", "            run += dt[t] * A[h];\n            cs[t] = run;",
     "            cs[t] = run;\n            run += dt[t] * A[h];"),
    ("chunked_offdiag_dropped", "yl[p] += e * acc;", "yl[p] += 0.0 * e * acc;"),
    ("chunked_state_decay_wrong", "const double w = exp(acs[len - 1] - acs[s]) * dt[s];",
     "const double w = exp(acs[len - 1]) * dt[s];"),
    ("softplus_bias_dropped", "const double dt = sp(dt_raw[(b * L + t) * H + h] + bias);",
     "const double dt = sp(dt_raw[(b * L + t) * H + h]);"),
    ("decode_state_not_decayed", "const double v = decay * st[n * P + p] + dt * Bt[n] * xt[p];",
     "const double v = st[n * P + p] + dt * Bt[n] * xt[p];"),
    ("mimo_input_reads_C", "for (int64_t r = 0; r < R; ++r) in += Bt[r * N + n] * Xt[r * P + p];",
     "for (int64_t r = 0; r < R; ++r) in += Ct[r * N + n] * Xt[r * P + p];"),
    ("mimo_only_first_rank", "for (int64_t r = 0; r < R; ++r) in += Bt[r * N + n] * Xt[r * P + p];",
     "for (int64_t r = 0; r < 1; ++r) in += Bt[r * N + n] * Xt[r * P + p];"),
    ("mimo_output_rank_swapped", "for (int64_t r = 0; r < R; ++r) yt[r * P + p] += Ct[r * N + n] * v;",
     "for (int64_t r = 0; r < R; ++r) yt[r * P + p] += Ct[(R - 1 - r) * N + n] * v;"),
    ("bwd_final_seed_dropped", "if (dfinal) memcpy(Gs, dfinal", "if (0) memcpy(Gs, dfinal"),
    ("bwd_adjoint_not_decayed", "for (int64_t i = 0; i < NP; ++i) Gs[i] *= decay;",
     "for (int64_t i = 0; i < NP; ++i) Gs[i] *= 1.0;"),
    ("bwd_softplus_derivative_dropped", "const double dz = ddt / (1.0 + exp(-z));", "const double dz = ddt;"),
    ("bwd_dB_missing_dt", "dBt[n] = dt * gx;", "dBt[n] = gx;"),
    ("bwd_dC_reads_previous_state", "hy += hc[n * P + p] * dyt[p];", "hy += hp[n * P + p] * dyt[p];"),
    ("bwd_decay_path_of_dt_dropped", "const double ddt = gbx + Ah * dlogdecay;", "const double ddt = gbx;"),
    ("m3_left_end_reads_current_token", "+= (1.0 - mix) * dt * Bp[n] * xp[p];", "+= (1.0 - mix) * dt * Bt[n] * xt[p];"),
    ("m3_left_end_weight_swapped", "+= (1.0 - mix) * dt * Bp[n] * xp[p];", "+= mix * dt * Bp[n] * xp[p];"),
    ("m3_rotation_not_orthogonal", "r0[p] = c * u - s * v;", "r0[p] = c * u + s * v;"),
    ("m3_angle_indexed_by_head", "const double ang = theta[((b * L + t) * G + g) * (N / 2) + k];",
     "const double ang = theta[((b * L + t) * G + h % G) * (N / 2) + k];"),
    ("m3_decode_buffers_not_advanced", "memcpy(x_prev, x, sizeof(double) * (size_t)(batch * H * P));", ";"),
    ("mimo_sequence_state_not_decayed", "st[n * P + p] = decay * st[n * P + p] + dt * in;",
     "st[n * P + p] = st[n * P + p] + dt * in;"),
    ("bwd_wrong_segment_checkpoint", "memcpy(seg, ck + k * NP, sizeof(double) * NP);",
     "memcpy(seg, ck + (k > 0 ? k - 1 : 0) * NP, sizeof(double) * NP);"),
]

PIN_TESTS = [
    lambda: pins.test_recurrent_equals_quadratic(2, True),
    lambda: pins.test_recurrent_equals_chunked(50, 16),
    pins.test_a_zero_is_causal_linear_attention,
    lambda: pins.test_dt_to_zero("recurrent"),
    lambda: pins.test_scalar_geometric_series("recurrent"),
    lambda: pins.test_scalar_geometric_series("quadratic"),
    lambda: pins.test_scalar_geometric_series("chunked"),
    lambda: pins.test_impulse_response_varying_dt("recurrent"),
    lambda: pins.test_impulse_response_varying_dt("quadratic"),
    lambda: pins.test_impulse_response_varying_dt("chunked"),
    pins.test_group_mapping,
    pins.test_decode_steps_equal_prefill,
    lambda: pins.test_mimo_step_is_a_chain_of_single_input_steps(2),
    lambda: pins.test_mimo_step_is_a_chain_of_single_input_steps(4),
    lambda: bwd_pins.test_backward_elementwise_finite_differences(2),
    lambda: bwd_pins.test_backward_directional_finite_differences(True, True),
    bwd_pins.test_backward_single_token_closed_form,
    lambda: m3_pins.test_mamba3_reduces_to_mamba2(True),
    m3_pins.test_trapezoid_impulse_response,
    m3_pins.test_trapezoid_step_response_closed_form,
    lambda: m3_pins.test_rotation_impulse_response(0.4),
    m3_pins.test_common_rotation_of_B_and_C_is_invisible,
    m3_pins.test_first_angle_acts_on_the_state_only,
    m3_pins.test_angles_follow_the_group_map,
    m3_pins.test_mamba3_decode_steps_equal_the_recurrence,
    lambda: pins.test_mimo_sequence_is_a_chain_of_mimo_steps(3),
]


def _load_mutant(tmp_path, name, old, new):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation {name}: anchor text not found"
    pkg = tmp_path / f"oracle_{name}"
    pkg.mkdir()
    init = open(os.path.join(ROOT, "oracle", "__init__.py")).read()
    (pkg / "__init__.py").write_text(init.replace('"-Werror",', ""))  # mutants may leave unused names
    (pkg / "ssd_oracle.c").write_text(src.replace(old, new, 1))
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", pkg / "__init__.py",
                                                  submodule_search_locations=[str(pkg)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name,old,new", MUTATIONS, ids=[m[0] for m in MUTATIONS])
def test_pins_catch_mutation(tmp_path, monkeypatch, name, old, new):
    mutant = _load_mutant(tmp_path, name, old, new)
    monkeypatch.setattr(pins, "oracle", mutant)
    monkeypatch.setattr(bwd_pins, "oracle", mutant)
    monkeypatch.setattr(m3_pins, "oracle", mutant)
    caught = 0
    for t in PIN_TESTS:
        try:
            t()
        except (AssertionError, ValueError):
            caught += 1
    assert caught > 0, f"no pin failed for mutation {name}"
