"""Plant plausible mistakes in copies of the C oracle and check that the pins catch every one.

Each mutant is one textual edit of ``oracle/gdn_oracle.c`` (a dropped term, a wrong sign, a wrong
index or head mapping, a transposed read, a wrong tap order, a wrong normalisation), compiled into
a temporary library on the CPU.  A mutant that passes all pins would mean the pins cannot tell that
mistake from the method, so the test fails.
"""
import os

import pytest

import oracle
import oracle_pins

MUTANTS = {
    "drop_beta_in_erase": ("x = S[(long)a * dk + c] - beta * Sk[a] * k[c];",
                           "x = S[(long)a * dk + c] - Sk[a] * k[c];"),
    "wrong_sign_erase": ("x = S[(long)a * dk + c] - beta * Sk[a] * k[c];",
                         "x = S[(long)a * dk + c] + beta * Sk[a] * k[c];"),
    "decay_also_on_write": ("S[(long)a * dk + c] = alpha * x + beta * v[a] * k[c];",
                            "S[(long)a * dk + c] = alpha * (x + beta * v[a] * k[c]);"),
    "drop_write_term": ("S[(long)a * dk + c] = alpha * x + beta * v[a] * k[c];",
                        "S[(long)a * dk + c] = alpha * x;"),
    "log_alpha_as_alpha": ("const double alpha = exp(J->log_alpha[(b * J->T + t) * Hv + h]);",
                           "const double alpha = 1.0 + J->log_alpha[(b * J->T + t) * Hv + h];"),
    "transposed_S0_read": ("J->S0[(((long)b * Hv + h) * dk + c) * dv + a]",
                           "J->S0[(((long)b * Hv + h) * dv + a) * dk + c]"),
    "transposed_S_T_write": ("J->S_T[(((long)b * Hv + h) * dk + c) * dv + a] =",
                             "J->S_T[(((long)b * Hv + h) * dv + a) * dk + c] ="),
    "gqa_interleaved_heads": ("const int hk = h / (Hv / Hk);", "const int hk = h % Hk;"),
    "erase_with_query": ("for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * k[c];\n"
                         "            Sk[a] = acc;",
                         "for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * q[c];\n"
                         "            Sk[a] = acc;"),
    "output_reads_key": ("for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * q[c];\n"
                         "            o[a] = J->scale * acc;",
                         "for (int c = 0; c < dk; ++c) acc += S[(long)a * dk + c] * k[c];\n"
                         "            o[a] = J->scale * acc;"),
    "output_ignores_scale": ("o[a] = J->scale * acc;", "o[a] = acc;"),
    "conv_taps_reversed": ("acc += w[c * 4 + j] * x[(b * T + s) * C + c];",
                           "acc += w[c * 4 + (3 - j)] * x[(b * T + s) * C + c];"),
    "conv_off_by_one": ("const long s = t - 3 + j;", "const long s = t - 4 + j;"),
    "conv_no_silu": ("y[(b * T + t) * C + c] = acc * sigmoid(acc);",
                     "y[(b * T + t) * C + c] = acc;"),
    "l2_eps_outside_sqrt": ("const double inv = 1.0 / sqrt(ss + eps);",
                            "const double inv = 1.0 / (sqrt(ss) + eps);"),
    "rms_sum_not_mean": ("const double inv = 1.0 / sqrt(ss / d + eps);",
                         "const double inv = 1.0 / sqrt(ss + eps);"),
    "gate_sigmoid_not_silu": ("* (zz * sigmoid(zz));", "* sigmoid(zz);"),
    "gain_ignored": ("y[r * d + i] = (o[r * d + i] * inv) * w[i] * (zz * sigmoid(zz));",
                     "y[r * d + i] = (o[r * d + i] * inv) * (zz * sigmoid(zz));"),
    # backward pass
    "bwd_output_grad_ignores_scale": ("G[(long)a * dk + c] += J->scale * dO[a] * q[c];",
                                      "G[(long)a * dk + c] += dO[a] * q[c];"),
    "bwd_dq_reads_previous_state": ("for (int a = 0; a < dv; ++a) acc += S[(long)a * dk + c] * dO[a];",
                                    "for (int a = 0; a < dv; ++a) acc += P[(long)a * dk + c] * dO[a];"),
    "bwd_dlog_alpha_missing_alpha": ("J->dla[row] = alpha * ga;", "J->dla[row] = ga;"),
    "bwd_dv_missing_beta": ("dvv[a] = beta * Gk[a];", "dvv[a] = Gk[a];"),
    "bwd_state_grad_not_decayed": ("for (long i = 0; i < SS; ++i) dP[i] = alpha * G[i];",
                                   "for (long i = 0; i < SS; ++i) dP[i] = G[i];"),
    "bwd_dbeta_drops_erase_term": ("db -= x[a] * acc;", "db -= 0.0 * acc;"),
    "bwd_dk_drops_state_term": ("dkk[c] += acc;", "dkk[c] += 0.0 * acc;"),
    "bwd_state_grad_drops_rank1": ("dP[(long)a * dk + c] += dx[a] * k[c];",
                                   "dP[(long)a * dk + c] += 0.0 * dx[a] * k[c];"),
    "bwd_silu_derivative_is_sigmoid": (
        "const double dpre = dy[(b * T + t) * C + c] * sg * (1.0 + pre * (1.0 - sg));",
        "const double dpre = dy[(b * T + t) * C + c] * sg;"),
    "bwd_conv_tap_reversed": ("dx[(b * T + u) * C + c] += w[c * 4 + j] * dpre;",
                              "dx[(b * T + u) * C + c] += w[c * 4 + 3 - j] * dpre;"),
    "bwd_l2_drops_projection": ("dx[r * d + i] = dy[r * d + i] / n - x[r * d + i] * xd / (n * n * n);",
                                "dx[r * d + i] = dy[r * d + i] / n;"),
    "bwd_rms_sum_not_mean": ("dout[r * d + i] = inv * g - o[r * d + i] * inv * inv * inv * go / d;",
                             "dout[r * d + i] = inv * g - o[r * d + i] * inv * inv * inv * go;"),
    "bwd_gate_a_sign": ("dba[r * 2 * Hv + Hv + h] = dlog_alpha[r * Hv + h] * sigmoid(-a);",
                        "dba[r * 2 * Hv + Hv + h] = dlog_alpha[r * Hv + h] * sigmoid(a);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(oracle.SOURCE).read()
    assert src.count(before) == 1, f"mutation site of {name} not unique in the oracle source"
    path = tmp_path / f"{name}.c"
    path.write_text(src.replace(before, after))
    lib = oracle.OracleLib(oracle.compile_source(str(path), str(tmp_path / f"{name}.so")))
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"no pin catches the mutant {name}"
