"""Each plausible mistake in the oracle trips at least one pin.

The oracle's C source is copied, one mistake is planted in the copy (on the
CPU, in a temporary directory), the copy is compiled, and every pin is run
against it.  A mutant that passes all pins would mean the pins cannot tell
that mistake from the formula.
"""
import os

import pytest

import oracle
from tests import oracle_bwd_pins, oracle_pins

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


# mistakes in the backward pass, each caught by a backward pin
BWD_MUTANTS = [
    ("delta_dropped", "dt[i * S + j] = p[i * S + j] * (dt[i * S + j] - delta);",
     "dt[i * S + j] = p[i * S + j] * (dt[i * S + j] - 0.0);"),
    ("dt_sign", "dt[i * S + j] = p[i * S + j] * (dt[i * S + j] - delta);",
     "dt[i * S + j] = p[i * S + j] * (delta - dt[i * S + j]);"),
    ("dp_from_keys", "dp += dO[i * D + d] * v[j * D + d];", "dp += dO[i * D + d] * k[j * D + d];"),
    ("dq_unscaled", "dq[i * D + d] = acc * inv_sqrt_d;", "dq[i * D + d] = acc;"),
    ("dk_unscaled", "dk[j * D + d] = acck * inv_sqrt_d;", "dk[j * D + d] = acck;"),
    ("dq_from_queries", "acc += dt[i * S + j] * k[j * D + d];", "acc += dt[i * S + j] * q[j * D + d];"),
    ("dk_transposed", "acck += dt[i * S + j] * q[i * D + d];", "acck += dt[j * S + i] * q[i * D + d];"),
    ("dv_from_dt", "accv += p[i * S + j] * dO[i * D + d];", "accv += dt[i * S + j] * dO[i * D + d];"),
    ("dv_transposed", "accv += p[i * S + j] * dO[i * D + d];", "accv += p[j * S + i] * dO[i * D + d];"),
    ("dmask_row_sums", "cs += dt[i * S + j];", "cs += dt[j * S + i];"),
    ("dpair_transposed", "dpair[e] += dt[e];", "dpair[e] += dt[(e % S) * S + e / S];"),
    ("dpair_weights", "dpair[e] += dt[e];", "dpair[e] += p[e];"),
    ("bwd_pair_transposed", "if (pair) tij += pair[i * S + j];", "if (pair) tij += pair[j * S + i];"),
    ("bwd_mask_dropped", "if (mask) tij += mask[j];", "if (mask) tij += 0.0;"),
    ("bwd_weights_unnormalised", "double pij = exp(p[i * S + j] - lse[i]);",
     "double pij = exp(p[i * S + j] - lse[i] + 0.5);"),
    ("rows_delta_dropped", "out[j] = out[j] * (dp[j] - delta);", "out[j] = out[j] * dp[j];"),
    ("rows_pair_transposed", "if (ps) tij += ps[j];",
     "if (ps) tij += pair[pair_mat[s] * S * S + j * S + i];"),
]


def _pins_that_catch(src, old, new, tmp_path, pins):
    assert old in src, "mutation site not found"
    mutated = tmp_path / "mutant.c"
    mutated.write_text(src.replace(old, new, 1))
    lib = oracle.compile_source(str(mutated), str(tmp_path / "libmutant.so"))
    orc = oracle.Oracle(lib)
    caught = []
    for pin in pins:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    return caught


@pytest.mark.parametrize("name,old,new", BWD_MUTANTS, ids=[m[0] for m in BWD_MUTANTS])
def test_bwd_mutant_is_caught(tmp_path, name, old, new):
    src = open(oracle.SOURCE).read()
    caught = _pins_that_catch(src, old, new, tmp_path, oracle_bwd_pins.ALL_BWD_PINS)
    assert caught, f"backward mutant {name} passed every backward pin"


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
