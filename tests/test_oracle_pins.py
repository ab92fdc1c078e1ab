"""The oracle against its pins, and the pins against planted mistakes.

Every pin in ``tests/oracle_pins.py`` must hold for the oracle.  Then each mutant
below (a plausible slip planted in a copy of the oracle's C source, compiled on the
CPU) must fail at least one pin: that shows the pins would catch it.
"""
import os
import shutil

import pytest

import oracle
from tests import oracle_pins


@pytest.fixture(scope="module")
def O():
    return oracle.default()


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda f: f.__name__)
def test_pin(O, pin):
    pin(O)


# (name, text in ref_attn.c, replacement)
MUTANTS = [
    ("head_mapping_modulo", "int kvh = h / g;", "int kvh = h % Hk;"),
    ("causal_strict", "return !causal || (long)j <= (long)i + (long)(Sk - Sq);",
     "return !causal || (long)j < (long)i + (long)(Sk - Sq);"),
    ("causal_top_left", "return !causal || (long)j <= (long)i + (long)(Sk - Sq);",
     "return !causal || (long)j <= (long)i;"),
    ("scale_dropped", "s[j - key_lo] = scale * dot;", "s[j - key_lo] = dot;"),
    ("lse_without_max", "*lse = m + log(l);", "*lse = log(l);"),
    ("lse_log2", "*lse = m + log(l);", "*lse = m + log2(l);"),
    ("values_from_keys", "const double* vj = v + (long)j * kv_row_stride;",
     "const double* vj = k + (long)j * kv_row_stride;"),
    ("no_normalisation", "for (int c = 0; c < d; ++c) o[c] /= l;", ""),
    ("max_not_subtracted_in_weights", "double p = exp(s[j - key_lo] - m);",
     "double p = exp(s[j - key_lo]);"),
    ("combine_weight_sign", "double w = exp(lse_parts[(long)s * rows + r] - M);",
     "double w = exp(M - lse_parts[(long)s * rows + r]);"),
    ("combine_lse_without_max", "lse[r] = M + log(wsum);", "lse[r] = log(wsum);"),
    ("key_range_lower_ignored", "if (key_lo < 0) key_lo = 0;", "key_lo = 0;"),
    ("key_range_upper_ignored", "if (key_hi > Sk) key_hi = Sk;", "key_hi = Sk;"),
    ("kv_row_stride_wrong", "gqa_oracle_row(qi, kb, vb, (long)Hk * d,", "gqa_oracle_row(qi, kb, vb, (long)d,"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new):
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, f"mutant {name}: pattern not found in the oracle source"
    mutated = src.replace(old, new)
    shutil.copy(oracle.HDR, tmp_path / "ref_attn.h")
    (tmp_path / "ref_attn.c").write_text(mutated)
    lib = tmp_path / f"liboracle_{name}.so"
    oracle.compile_oracle(str(tmp_path / "ref_attn.c"), str(lib), str(tmp_path))
    M = oracle.Oracle(str(lib))
    failed = []
    for pin in oracle_pins.PINS:
        try:
            pin(M)
        except (AssertionError, ValueError, FloatingPointError):
            failed.append(pin.__name__)
    assert failed, f"no pin caught the planted mistake {name}"
