"""Plant plausible mistakes in copies of oracle.c and check that a pin catches each.

Every mutant is compiled from a textual edit of the oracle source into a
temporary directory; the committed oracle is never touched.  A mutant that
survived every pin would mean the pins cannot tell that slip from the truth.
"""
import os
import shutil
import subprocess

import pytest

import oracle
from test_oracle_pins import ALL_PINS

MUTANTS = {
    "transposed_W_index": ("Wt[j * ldw + p]", "Wt[p * ldw + j]"),
    "dropped_last_term": ("p < k; ++p", "p < k - 1; ++p"),
    "wrong_sign": ("acc += prod;", "acc -= prod;"),
    "S_without_abs": ("mag += fabs(prod);", "mag += prod;"),
    "bf16_bias_off_by_one": ("e - 127);", "e - 126);"),
    "f16_subnormal_scale": ("ldexp((double)f, -14 - 10)", "ldexp((double)f, -14 - 9)"),
    "bf16_fraction_width": ("(double)f / 128.0", "(double)f / 256.0"),
    "topk_ties_higher_index": ("(x->i < y->i) ? -1 : (x->i > y->i)",
                               "(x->i > y->i) ? -1 : (x->i < y->i)"),
    "topk_ascending": ("if (x->v > y->v) return -1;", "if (x->v < y->v) return -1;"),
    "nan_ranked_last": ("return xn ? -1 : 1;", "return xn ? 1 : -1;"),
    "ulp_f16_fraction_bits": ("(e - 1) - 10)", "(e - 1) - 11)"),
    "ulp_bf16_binade": ("(e - 1) - 7)", "e - 7)"),
    "bf16_ties_away": ("lower > 0x8000u || (lower == 0x8000u && (upper & 1u))", "lower >= 0x8000u"),
    "bf16_truncate": ("upper += 1u;", "upper += 0u;"),
    "sigmoid_sign": ("1.0 / (1.0 + exp(-x))", "1.0 / (1.0 + exp(x))"),
    "float_accumulator": ("double acc = 0.0, mag = 0.0;", "float acc = 0.0f, mag = 0.0f;"),
    "descending_k": ("for (int64_t p = 0; p < k; ++p) {", "for (int64_t p = k - 1; p >= 0; --p) {"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    if shutil.which("gcc") is None:
        pytest.skip("gcc not available")
    old, new = MUTANTS[name]
    src = open(oracle.SRC).read()
    assert src.count(old) >= 1, f"mutation site for {name} not found"
    mutated = src.replace(old, new)
    msrc = tmp_path / "oracle_mutant.c"
    msrc.write_text(mutated)
    mlib = str(tmp_path / "liboracle_mutant.so")
    oracle.build(force=True, src=str(msrc), out=mlib)
    orc = oracle.Oracle(mlib)
    caught = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            caught.append(pin.__name__)
    assert caught, f"mutant {name} passed every pin"
