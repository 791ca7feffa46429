"""Plants plausible mistakes in copies of the oracle (on the CPU) and checks
that at least one pin catches each of them.  The oracle source itself is never
modified: each mutant is a temporary copy compiled into its own library.
"""
import os
import shutil

import pytest

from oracle import oracle as O
from tests.oracle_pins import PINS

MUTANTS = {
    "dropped_scale": ("s[j] = J->scale * dot(qi, J->k + j * J->d, J->d);",
                      "s[j] = dot(qi, J->k + j * J->d, J->d);"),
    "transposed_scores": ("s[j] = J->scale * dot(qi, J->k + j * J->d, J->d);",
                          "s[j] = J->scale * dot(J->q + j * J->d, J->k + i * J->d, J->d);"),
    "causal_off_by_one": ("int64_t v = i + 1 + (nk - nq);", "int64_t v = i + (nk - nq);"),
    "causal_top_left": ("int64_t v = i + 1 + (nk - nq);", "int64_t v = i + 1;"),
    "masked_row_sees_a_key": ("return v < 0 ? 0 : (v > nk ? nk : v);", "return v < 1 ? 1 : (v > nk ? nk : v);"),
    "lse_without_max": ("return m + log(l);", "return log(l);"),
    "values_from_keys": ("const double *vj = J->v + j * J->d;\n            for (int64_t c = 0; c < J->d; ++c) o[c] += p * vj[c];",
                         "const double *vj = J->k + j * J->d;\n            for (int64_t c = 0; c < J->d; ++c) o[c] += p * vj[c];"),
    "dropped_D_term": ("double dsij = s[j] * (ds[j] - D);", "double dsij = s[j] * ds[j];"),
    "dq_missing_scale": ("for (int64_t c = 0; c < J->d; ++c) dq[c] *= J->scale;", ""),
    "dk_wrong_operand": ("dk[c] += dsij * qi[c];", "dk[c] += dsij * doi[c];"),
    "dv_uses_dS": ("dv[c] += p * doi[c];", "dv[c] += dsij * doi[c];"),
    "dk_missing_scale": ("for (int64_t c = 0; c < J->d; ++c) dk[c] *= J->scale;", ""),
    "dkdv_causal_range": ("int64_t i0 = J->causal ? j - (J->nk - J->nq) : 0;",
                          "int64_t i0 = J->causal ? j + 1 - (J->nk - J->nq) : 0;"),
    "dkdv_top_left": ("int64_t i0 = J->causal ? j - (J->nk - J->nq) : 0;", "int64_t i0 = J->causal ? j : 0;"),
    "dP_wrong_sign": ("double dsij = p * (dp - J->dsum_all[i]);", "double dsij = p * (J->dsum_all[i] - dp);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(O._SRC).read()
    old, new = MUTANTS[name]
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new, 1)
    path = tmp_path / "mutant.c"
    path.write_text(mutated)
    lib = O.load(O.build(force=True, src=str(path), out=str(tmp_path / "libmutant.so")))
    caught = []
    for pin in PINS:
        try:
            pin(lib)
        except (AssertionError, RuntimeError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
    shutil.rmtree(tmp_path, ignore_errors=True)
