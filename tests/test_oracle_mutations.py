"""Plant plausible mistakes in copies of the oracle source and check that at
least one pin fails for each.  This shows the pins constrain every part of
the oracle: a dropped term, a flipped sign, a wrong index or a transposed
operand anywhere in it is caught.  Mistakes are planted only in the CPU
oracle, never in GPU code."""
import os

import pytest

import oracle
import oracle_pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pararnn_oracle.c")

MUTATIONS = {
    "linear_swapped_gates": ("out[0] = p[0] * s[0] + p[1];", "out[0] = p[1] * s[0] + p[0];"),
    "gru_step_sign": ("out[0] = (1.0 - z) * h + z * c;", "out[0] = (1.0 - z) * h - z * c;"),
    "gru_reset_gate_dropped": ("double c = tanh(p[2] + w[2] * r * h);\n        out[0]",
                               "double c = tanh(p[2] + w[2] * h);\n        out[0]"),
    "gru_jacobian_term_dropped": ("A[0] = (1.0 - z) + w[0] * Gz + w[1] * Gr + w[2] * r * Gc;",
                                  "A[0] = (1.0 - z) + w[0] * Gz + w[2] * r * Gc;"),
    "lstm_forget_bias_dropped": ("double fg = sig(p[1] + w[1] * h + 1.0);\n        double og = sig(p[2] + w[2] * h);\n"
                                 "        double gg = tanh(p[3] + w[3] * h);\n        double cn = fg * c + ig * gg;\n"
                                 "        out[0] = cn;",
                                 "double fg = sig(p[1] + w[1] * h);\n        double og = sig(p[2] + w[2] * h);\n"
                                 "        double gg = tanh(p[3] + w[3] * h);\n        double cn = fg * c + ig * gg;\n"
                                 "        out[0] = cn;"),
    "lstm_jacobian_transposed": ("A[1] = dcn_dh;                               /* dc'/dh */\n"
                                 "        A[2] = og * (1.0 - tn * tn) * fg;            /* dh'/dc */",
                                 "A[2] = dcn_dh;\n        A[1] = og * (1.0 - tn * tn) * fg;"),
    "lstm_output_gate_grad": ("dh[2] = og * (1.0 - og) * tn;", "dh[2] = og * (1.0 - og);"),
    "newton_sign": ("double acc = -F;", "double acc = F;"),
    "newton_wrong_linearisation_point": ("oracle_cell_jacobian(j->cell, p, w, prev_old, A);\n            for (int i = 0; i < S; ++i) {\n                double F",
                                         "oracle_cell_jacobian(j->cell, p, w, cur_old, A);\n            for (int i = 0; i < S; ++i) {\n                double F"),
    "newton_no_warm_start": ("oracle_cell_step(j->cell, p, w, zero, fv);\n        for (int i = 0; i < S; ++i) *Hat(j->H, j, b, t, i, d) = fv[i];",
                             "for (int i = 0; i < S; ++i) *Hat(j->H, j, b, t, i, d) = 0.0;"),
    "adjoint_transposed": ("for (int m = 0; m < S; ++m) nl[i] += A[m * S + i] * lam[m];",
                           "for (int m = 0; m < S; ++m) nl[i] += A[i * S + m] * lam[m];"),
    "adjoint_wrong_time_index": ("load_p(j, b, t + 1, d, pn);", "load_p(j, b, t, d, pn);"),
    "adjoint_da_uses_dp": ("ga += lam[i] * da[i * G + g];", "ga += lam[i] * dp[i * G + g];"),
    "picard_forward_order": ("for (int64_t t = j->T - 1; t >= 0; --t) {\n            load_p(j, b, t, d, p);\n            if (t > 0)",
                             "for (int64_t t = 0; t < j->T; ++t) {\n            load_p(j, b, t, d, p);\n            if (t > 0)"),
    "picard_sweep_skipped": ("for (int sweep = 0; sweep < j->P; ++sweep) {", "for (int sweep = 1; sweep < j->P; ++sweep) {"),
    "picard_zero_initial_state": ("            else\n                load_h0(j, b, d, prev);\n            oracle_cell_step(j->cell, p, w, prev, fv);",
                                  "            else\n                prev[0] = prev[1] = 0.0;\n            oracle_cell_step(j->cell, p, w, prev, fv);"),
    "residual_wrong_row": ("cur[i] = Hget(j->H, j, b, t, i, d);", "cur[i] = Hget(j->H, j, b, t > 0 ? t - 1 : 0, i, d);"),
    # head-wise GRU
    "head_step_weight_transposed": ("            az += Uz[(size_t)i * d + j] * s[j];\n            ar += Ur[(size_t)i * d + j] * s[j];\n"
                                    "            n += Uc[(size_t)i * d + j] * s[j];\n        }\n"
                                    "        double z = sig(az), r = sig(ar), c = tanh(p[2 * d + i] + r * n);\n        out[i]",
                                    "            az += Uz[(size_t)j * d + i] * s[j];\n            ar += Ur[(size_t)i * d + j] * s[j];\n"
                                    "            n += Uc[(size_t)i * d + j] * s[j];\n        }\n"
                                    "        double z = sig(az), r = sig(ar), c = tanh(p[2 * d + i] + r * n);\n        out[i]"),
    "head_reset_gate_dropped": ("c = tanh(p[2 * d + i] + r * n);\n        out[i]", "c = tanh(p[2 * d + i] + n);\n        out[i]"),
    "head_jacobian_term_dropped": ("beta * Ur[(size_t)i * d + j] +", "0.0 * Ur[(size_t)i * d + j] +"),
    "head_jacobian_transposed": ("A[(size_t)i * d + j] = (i == j ? 1.0 - z : 0.0)", "A[(size_t)j * d + i] = (i == j ? 1.0 - z : 0.0)"),
    "head_newton_sign": ("double acc = -F[i];", "double acc = F[i];"),
    "head_newton_linearised_at_new_iterate": (
        "memcpy(prev, s + t * d, d * sizeof(double));   /* s^(k)_t, the next row's s_{t-1} */\n"
        "                if (k < j->K)\n                    for (int i = 0; i < d; ++i) s[t * d + i] += del[i];",
        "if (k < j->K)\n                    for (int i = 0; i < d; ++i) s[t * d + i] += del[i];\n"
        "                memcpy(prev, s + t * d, d * sizeof(double));"),
    "head_no_warm_start": ("oracle_head_gru_step(d, p, U, tmp, s + t * d);",
                           "for (int i = 0; i < d; ++i) s[t * d + i] = 0.0;"),
    "head_adjoint_transposed": ("for (int i = 0; i < d; ++i) acc += A[(size_t)i * d + m] * lam[i];",
                                "for (int i = 0; i < d; ++i) acc += A[(size_t)m * d + i] * lam[i];"),
    "head_adjoint_dUc_factor": ("+= lam[i] * ga[i] * prev[m];", "+= lam[i] * be[i] * prev[m];"),
    "head_adjoint_state_index": ("prev[i] = j->H[(b * T + t - 1) * j->D + (int64_t)h * d + i];",
                                 "prev[i] = j->H[(b * T + t) * j->D + (int64_t)h * d + i];"),
    "head_adjoint_dpc_factor": ("j->dpx[o + 2 * j->D] = lam[i] * zc[i];", "j->dpx[o + 2 * j->D] = lam[i] * ga[i];"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, "mutation anchor for %s not found exactly once" % name
    mutant_c = tmp_path / "mutant.c"
    mutant_c.write_text(src.replace(old, new))
    so = oracle.compile_source(str(mutant_c), str(tmp_path / "libmutant.so"))
    caught = []
    with oracle.use_library(so):
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except AssertionError as e:
                caught.append("%s: %s" % (pin.__name__, str(e).splitlines()[0] if str(e) else ""))
            except Exception as e:  # a mutant may also crash a pin's arithmetic
                caught.append("%s raised %s" % (pin.__name__, type(e).__name__))
    assert caught, "no pin caught mutation %s" % name
