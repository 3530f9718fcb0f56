"""Plant plausible mistakes in a copy of the oracle (on the CPU) and check that the pins catch each.

Every mutant is one textual change to ``oracle/oracle.c`` compiled into a temporary library; a
mutant that passes every pin would mean the pins leave that part of the oracle unchecked.
"""
import os
import subprocess

import pytest

import oracle
from oracle_pins import PINS

SRC = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle", "oracle.c")

MUTANTS = {
    "round_half_away": ("nearbyint(", "round("),
    "scale_over_128": ("amax / 127.0f", "amax / 128.0f"),
    "zero_row_scale": ("*s = 1.0f;", "*s = 0.0f;"),
    "silu_sign": ("a1 / (1.0 + exp(-a1)) * a3", "a1 / (1.0 + exp(a1)) * a3"),
    "dropped_up_proj": ("a1 / (1.0 + exp(-a1)) * a3", "a1 / (1.0 + exp(-a1))"),
    "gate_scale_for_up": ("sc3 = (double)s3[j]", "sc3 = (double)s1[j]"),
    "down_transposed": ("((double)r2[j] * sc2)", "((double)q2[j * d + i] * sc2)"),
    "tie_to_higher_index": ("z[e] > z[best]", "z[e] >= z[best]"),
    "bias_sign": ("acc += (double)bias[e];", "acc -= (double)bias[e];"),
    "softmax_unnormalised": ("p[e] /= denom;", "(void)denom;"),
    "dropped_gate_weight": ("yt[i] += wts[k] * o[i];", "yt[i] += o[i];"),
    "bf16w_down_transposed": ("acc += (double)bf16_value(r2[j]) * h[j];",
                              "acc += (double)bf16_value(w2[j * d + i]) * h[j];"),
    "bf16w_up_uses_gate": ("a3 += (double)bf16_value(r3[i]) * xd[i];", "a3 += (double)bf16_value(r1[i]) * xd[i];"),
    "mlp_ignores_token_list": ("c->tokens[n] : n;\n        const uint16_t* xt = c->x + t * d;\n        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);\n        expert_ffn",
                               "n : n;\n        const uint16_t* xt = c->x + t * d;\n        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);\n        expert_ffn"),
    "mlp_first_token_only": ("xt = c->x + t * d;\n        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);\n        expert_ffn",
                             "xt = c->x;\n        for (int64_t i = 0; i < d; ++i) xd[i] = (double)bf16_value(xt[i]);\n        expert_ffn"),
    "fp8_scale_over_512": ("amax / 448.0f", "amax / 512.0f"),
    "fp8_ties_away": ("nearbyint(ldexp(a, 3 - eb))", "round(ldexp(a, 3 - eb))"),
    "fp8_flush_subnormals": ("if (eb < -6) eb = -6;", "if (eb < -6) return sign;"),
    "fp8_h_not_quantized": ("(e4m3_value(h8[j]) * (double)hs)", "h[j]"),
    "fp8_h_not_bf16": ("e4m3_round(bf16_round((float)h[j]) / (double)hs)", "e4m3_round(h[j] / (double)hs)"),
    "fp8_x_not_quantized": ("xd[i] = e4m3_value(xq[i]) * (double)xs;", "xd[i] = (double)bf16_value(xt[i]);"),
    "router_ignores_last_input": ("for (int64_t i = 0; i < d; ++i) acc += (double)bf16_value(x[i])",
                                  "for (int64_t i = 0; i + 1 < d; ++i) acc += (double)bf16_value(x[i])"),
}


def _build_mutant(name, tmp_path):
    # every mutant must keep all memory accesses in bounds: it runs inside the test process
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-shared", "-fPIC", "-pthread", str(c), "-o", str(so), "-lm"])
    return oracle.Oracle(str(so))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    orc = _build_mutant(name, tmp_path)
    failed = []
    for pin in PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
