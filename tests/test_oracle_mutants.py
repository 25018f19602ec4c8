"""The pins are strong enough: every plausible slip planted in a copy of the oracle
(a dropped term, a wrong sign or index, a transposed operand) fails at least one pin.

Each mutant is the oracle's C source with one textual substitution, compiled with
gcc into a temporary library; the oracle itself is never modified.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from oracle_pins import ALL_PINS

MUTANTS = {
    "decay_exponent_off_by_one": ("exp(-(double)(t - 1 - i) * w[c]", "exp(-(double)(t - i) * w[c]"),
    "direct_drops_bonus": ("double e = exp(u[c] + k[at3(b, t, c, T, C)]);",
                           "double e = exp(k[at3(b, t, c, T, C)]);"),
    "direct_includes_current_in_past": ("for (int64_t i = 0; i < t; ++i)", "for (int64_t i = 0; i <= t; ++i)"),
    "direct_drops_current_value": ("num += e * v[at3(b, t, c, T, C)];", "num += e;"),
    "output_max_ignores_bonus": ("double q = fmax(p, u[c] + kt);", "double q = fmax(p, kt);"),
    "update_decay_sign": ("double p_new = fmax(p - w[c], kt);", "double p_new = fmax(p + w[c], kt);"),
    "update_drops_decay": ("double keep = exp(p - w[c] - p_new);", "double keep = exp(p - p_new);"),
    "update_drops_value": ("a = keep * a + add * vt;", "a = keep * a + add;"),
    "denominator_gets_value": ("bb = keep * bb + add;", "bb = keep * bb + add * vt;"),
    "output_transposed_operand": ("(w_past * a + w_now * vt) / den", "(w_past * bb + w_now * vt) / den"),
    "output_bonus_on_past": ("double w_now = exp(u[c] + kt - q);", "double w_now = exp(kt - q);"),
    "naive_decay_sign": ("double decay = exp(-w[c]);", "double decay = exp(w[c]);"),
    "naive_update_before_output": ("a = decay * a + exp(kt) * vt;", "a = a + exp(kt) * vt;"),
    "state_in_swaps_b_p": ("bb = state_in[BC + bc];", "bb = state_in[2 * BC + bc];"),
    "state_out_drops_p": ("state_out[2 * BC + bc] = p;", "state_out[2 * BC + bc] = 0.0;"),
    "lerp_weight_swapped": ("(1.0 - mu[c]) * prev", "mu[c] * prev"),
    "lerp_previous_token_index": ("prev = x[at3(b, t - 1, c, T, C)];", "prev = x[at3(b, t, c, T, C)];"),
    "layout_transposed": ("return ((size_t)b * (size_t)T + (size_t)t) * (size_t)C + (size_t)c;",
                          "return ((size_t)b * (size_t)C + (size_t)c) * (size_t)T + (size_t)t;"),
    "magnitude_scale_signed": ("sa = keep * sa + add * fabs(vt);", "sa = keep * sa + add * vt;"),
    "gate_sign": ("const double sigma = 1.0 / (1.0 + exp(-r[i]));", "const double sigma = 1.0 / (1.0 + exp(r[i]));"),
    "gate_offset": ("const double sigma = 1.0 / (1.0 + exp(-r[i]));", "const double sigma = 1.0 / (2.0 + exp(-r[i]));"),
    "gate_divides": ("out[i] = wkv[i] * sigma;", "out[i] = wkv[i] / sigma;"),
    "backward_drops_current_value": ("gv[at3(b, t, c, T, C)] += g * alpha;", "gv[at3(b, t, c, T, C)] += 0.0 * alpha;"),
    "backward_key_uses_own_output": ("gk[at3(b, i, c, T, C)] += g * beta * (vi - yt);",
                                     "gk[at3(b, i, c, T, C)] += g * beta * vi;"),
    "backward_decay_count_off_by_one": ("gwc += -g * (double)(t - 1 - i) * beta * (vi - yt);",
                                        "gwc += -g * (double)(t - i) * beta * (vi - yt);"),
    "backward_bonus_sign": ("guc += g * alpha * (vt - yt);", "guc += g * alpha * (yt - vt);"),
    "eagle_decay_on_value_index": ("const double d = exp(-w[h * N + m]);\n                    const double km",
                                   "const double d = exp(-w[h * N]);\n                    const double km"),
    "eagle_outer_product_transposed": ("S[m * N + j] = d * S[m * N + j] + km * vj;",
                                       "S[j * N + m] = d * S[j * N + m] + km * vj;"),
    "eagle_drops_current_token": ("S[m * N + j] = d * S[m * N + j] + km * vj;", "S[m * N + j] = d * S[m * N + j];"),
    "eagle_readout_transposed": ("acc += rm * S[m * N + j];", "acc += rm * S[j * N + m];"),
    "eagle_decay_sign": ("const double d = exp(-w[h * N + m]);", "const double d = exp(w[h * N + m]);"),
    "eagle_head_offset": ("const double rm = r[at3(b, t, h * N + m, T, C)];\n                        acc += rm * S",
                          "const double rm = r[at3(b, t, m, T, C)];\n                        acc += rm * S"),
    "eagle_state_in_transposed": ("S[e] = state_in ? state_in[sb + e] : 0.0;",
                                  "S[e] = state_in ? state_in[sb + (e % N) * N + e / N] : 0.0;"),
    "eagle_direct_decay_off_by_one": ("exp(-(double)(t - i) * w[h * N + m])", "exp(-(double)(t - 1 - i) * w[h * N + m])"),
    "eagle_direct_state_in_undecayed": ("exp(-(double)(t + 1) * w[h * N + m]) * state_in",
                                        "exp(-(double)t * w[h * N + m]) * state_in"),
    "eagle_scale_inflated": ("acc_s += fabs(rm) * Sa[m * N + j];", "acc_s += 1000.0 * fabs(rm) * Sa[m * N + j];"),
    "eagle_scale_state_signed": ("Sa[m * N + j] = d * Sa[m * N + j] + fabs(km) * fabs(vj);",
                                 "Sa[m * N + j] = d * Sa[m * N + j] + km * vj;"),
    "backward_sk_inflated": ("if (sk) sk[at3(b, i, c, T, C)] += gm * beta * (fabs(vi) + fabs(yt));",
                             "if (sk) sk[at3(b, i, c, T, C)] += 1000.0 * gm * beta * (fabs(vi) + fabs(yt));"),
    "backward_sv_inflated": ("if (sv) sv[at3(b, t, c, T, C)] += gm * alpha;",
                             "if (sv) sv[at3(b, t, c, T, C)] += 1000.0 * gm * alpha;"),
    "backward_sw_inflated": ("swc += gm * (double)(t - 1 - i) * beta * (fabs(vi) + fabs(yt));",
                             "swc += 1000.0 * gm * (double)(t - 1 - i) * beta * (fabs(vi) + fabs(yt));"),
    "backward_su_inflated": ("suc += gm * alpha * (fabs(vt) + fabs(yt));", "suc += 1000.0 * gm * alpha * (fabs(vt) + fabs(yt));"),
    "backward_scale_difference": ("if (sk) sk[at3(b, i, c, T, C)] += gm * beta * (fabs(vi) + fabs(yt));",
                                  "if (sk) sk[at3(b, i, c, T, C)] += gm * beta * fabs(vi - yt);"),
}


def _failing_pins(lib):
    failed = []
    for pin in ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    return failed


@pytest.mark.skipif(shutil.which("gcc") is None, reason="gcc needed to build mutants")
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutant_src = tmp_path / "mutant.c"
    mutant_src.write_text(src.replace(old, new))
    so = tmp_path / "libmutant.so"
    oracle.build(force=True, src=str(mutant_src), out=str(so))
    lib = oracle.load(str(so))
    assert _failing_pins(lib), f"mutant {name} passed every pin"
