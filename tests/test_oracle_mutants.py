"""Plant mistakes in copies of the oracle and check that the pins catch them.

Each mutant is a one-line change to ``oracle/avq_oracle.c`` of the kind a
reader could plausibly make (a flipped comparison, a dropped term, a wrong
sign or index, a transposed operand). It is compiled on the CPU into a
temporary library; the test passes only if at least one pin fails on it.
"""
import os

import pytest

import oracle_pins as pins
from oracle import oracle as orc

MUTANTS = {
    "child_reassign_on_tie": ("if (dd < leaf_d)", "if (dd <= leaf_d)"),
    "parent_tie_to_highest": ("if (dd < best)", "if (dd <= best)"),
    "parent_stats_stay_only": ("cnt[parent] += 1;\n            for (int j = 0; j < d; ++j) vs[(int64_t)parent * d + j] += v[j];",
                               "if (leaf == parent) { cnt[parent] += 1;\n            for (int j = 0; j < d; ++j) vs[(int64_t)parent * d + j] += v[j]; }"),
    "child_layout_transposed": ("int idx = M0 + best_p * C + c;", "int idx = M0 + c * M0 + best_p;"),
    "importance_without_count": ("s += A[r * M0 + p] * (double)cnt[p] / Zbar[r];", "s += A[r * M0 + p] / Zbar[r];"),
    "importance_without_normaliser": ("s += A[r * M0 + p] * (double)cnt[p] / Zbar[r];", "s += A[r * M0 + p] * (double)cnt[p];"),
    "zbar_without_count": ("z += a * (double)cnt[p];", "z += a;"),
    "select_smallest": ("if (w[a] > w[b]) return 1;\n    if (w[a] < w[b]) return 0;",
                        "if (w[a] < w[b]) return 1;\n    if (w[a] > w[b]) return 0;"),
    "delta_sign_flipped": ("const double dA = exp(Sc[j * C + c] - M) - ep;", "const double dA = ep - exp(Sc[j * C + c] - M);"),
    "correction_denominator_dropped": ("den += dA * (double)cnt[idx];", ""),
    "child_logit_unscaled": ("double s = scale * dot(q, cb + (int64_t)idx * d, d);", "double s = dot(q, cb + (int64_t)idx * d, d);"),
    "child_of_wrong_parent": ("const int idx = M0 + p * C + c;\n                double s", "const int idx = M0 + ((p + 1) % M0) * C + c;\n                double s"),
    "parent_logit_query_transposed": ("S[r * M0 + p] = scale * dot(q, cb + (int64_t)p * d, d);",
                                      "S[r * M0 + p] = scale * dot(Qbh + (int64_t)(i0 + p % rows) * d, cb + (int64_t)r * d, d);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    with open(orc.SRC) as f:
        src = f.read()
    assert src.count(old) >= 1, f"mutation anchor not found for {name}"
    mutated = src.replace(old, new, 1)
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(mutated)
    lib = orc.build(path, os.path.join(tmp_path, "libmutant.so"))
    m = orc.Oracle(lib)
    caught = []
    for pin in pins.ALL_PINS:
        try:
            pin(m)
        except (AssertionError, RuntimeError, IndexError, ValueError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught mutant {name}"
