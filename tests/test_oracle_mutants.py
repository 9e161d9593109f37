"""Each plausible mistake in the oracle trips at least one pin.

The oracle's C source is copied, one mistake is planted in the copy (on the
CPU, in a temporary directory), the copy is compiled, and every pin is run
against it.  A mutant that passes all pins would mean the pins cannot tell
that mistake from the formula.
"""
import os

import pytest

import oracle
from tests import oracle_pins

# (name, text in evo_oracle.c, replacement)
MUTANTS = [
    ("mask_subtracted", "if (mask) tj += mask[j];", "if (mask) tj -= mask[j];"),
    ("mask_dropped", "if (mask) tj += mask[j];", "if (mask) tj += 0.0;"),
    ("pair_dropped", "if (pair) tj += pair[i * S + j];", "if (pair) tj += 0.0;"),
    ("pair_transposed", "if (pair) tj += pair[i * S + j];", "if (pair) tj += pair[j * S + i];"),
    ("scale_one_over_d", "1.0 / sqrt((double)D)", "1.0 / (double)D"),
    ("no_scale", "1.0 / sqrt((double)D)", "1.0"),
    ("scale_on_biases_too", "t[j] = tj;\n        if (tj > m) m = tj;",
     "tj = tj / sqrt((double)D) * sqrt((double)D) * inv_sqrt_d / inv_sqrt_d; tj = (tj - dot * inv_sqrt_d) * inv_sqrt_d + dot * inv_sqrt_d;\n        t[j] = tj;\n        if (tj > m) m = tj;"),
    ("lse_without_max", "*lse_row = m + log(l);", "*lse_row = log(l);"),
    ("no_normalisation", "acc += (t[j] / l) * v[j * D + d];", "acc += t[j] * v[j * D + d];"),
    ("key_index_from_query", "dot += q[i * D + d] * k[j * D + d];", "dot += q[i * D + d] * k[i * D + d];"),
    ("value_transposed", "acc += (t[j] / l) * v[j * D + d];", "acc += (t[j] / l) * v[d * S + j];"),
    ("max_not_subtracted_in_lse", "t[j] = exp(t[j] - m);", "t[j] = exp(t[j] - m + 1.0);"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    assert old in src, f"mutation site for {name} not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = oracle.compile_source(str(mutated), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
