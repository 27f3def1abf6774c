"""Plant plausible mistakes in a copy of the oracle and check that at least
one pin fails for each.  The copy is compiled to a temporary library; the
oracle itself is untouched.  Each mutation names the exact source text it
replaces, so this test breaks loudly if the oracle is rewritten."""
import os

import pytest

from oracle import oracle as orc
from test_oracle_pins import PINS

SRC = os.path.join(os.path.dirname(orc.__file__), "retention_oracle.c")

MUTANTS = {
    # carried-state factor gamma^{j+1} off by one
    "xi_off_by_one": ("double xi = pow(g, (double)(j + 1));\n            for (int c = 0; c < dv; ++c) {\n                double s = 0.0;\n                for (int i = 0; i < dk; ++i) s += qj[i]",
                      "double xi = pow(g, (double)(j));\n            for (int c = 0; c < dv; ++c) {\n                double s = 0.0;\n                for (int i = 0; i < dk; ++i) s += qj[i]"),
    # a ragged last chunk decayed by the nominal chunk length
    "ragged_decay": ("double gn = pow(g, (double)n);", "double gn = pow(g, (double)chunk);"),
    # rotation turned the other way (conjugate on both rows)
    "rotation_sign": ("double c = cos(pos * theta), s = sin(pos * theta);",
                      "double c = cos(pos * theta), s = -sin(pos * theta);"),
    # frequency schedule base^(-j/d) instead of base^(-2j/d)
    "theta_formula": ("pow(theta_base, -2.0 * (double)j / (double)d)",
                      "pow(theta_base, -1.0 * (double)j / (double)d)"),
    # transposed scores in the parallel form
    "transposed_scores": ("dot(q + (size_t)t * dk, k + (size_t)m * dk, dk)",
                          "dot(q + (size_t)m * dk, k + (size_t)t * dk, dk)"),
    # decay dropped from the recurrence
    "no_state_decay": ("S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j] + k[i] * v[j];",
                       "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] + k[i] * v[j];"),
    # sigmoid gate instead of swish
    "sigmoid_gate": ("double sw = gv / (1.0 + exp(-gv));", "double sw = 1.0 / (1.0 + exp(-gv));"),
    # unbiased variance in GroupNorm
    "unbiased_var": ("var /= dv;", "var /= (dv - 1);"),
    # zeta applied as gamma^{j'} instead of gamma^{n-1-j'}
    "zeta_index": ("double zeta = pow(g, (double)(n - 1 - jj));", "double zeta = pow(g, (double)(jj));"),
    # normalisation gradient without the variance term
    "gn_grad_no_var_term": ("dO[orow + c] = r * (dn[c] - mean_dn - n[c] * mean_dnn);",
                            "dO[orow + c] = r * (dn[c] - mean_dn);"),
    # swish derivative taken as sigmoid(g) alone
    "swish_grad": ("dG[gy + c] = dY[gy + c] * n[c] * sig * (1.0 + gv * (1.0 - sig));",
                   "dG[gy + c] = dY[gy + c] * n[c] * sig;"),
    # gamma schedule 1 - 2^(-4-h)
    "gamma_schedule": ("gamma[h] = 1.0 - pow(2.0, -5.0 - (double)h);",
                       "gamma[h] = 1.0 - pow(2.0, -4.0 - (double)h);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path, olib):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not found exactly once"
    mut = tmp_path / f"{name}.c"
    mut.write_text(src.replace(old, new))
    lib = orc.load(orc.build(str(mut), str(tmp_path / f"lib{name}.so")))
    failed = []
    for pin in PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
