"""Sensitivity of the oracle pins: plant one plausible mistake at a time in a
copy of the oracle's C source (on the CPU), rebuild it, and check that at least
one pin from test_oracle.py fails.  The shipped oracle is never modified."""
import ctypes
import subprocess
from pathlib import Path

import numpy as np
import pytest

import oracle
from tests import test_oracle as pins
from tests import test_oracle_v2 as pins_v2

SRC = Path(oracle.__file__).resolve().parent / "tcsl_ref.c"

MUTANTS = {
    "value_index_halves_swapped": ("words[w++] = (uint32_t)v | (loc << 16);",
                                   "words[w++] = ((uint32_t)v << 16) | loc;"),
    "column_major_loc": ("uint32_t loc = (uint32_t)(r * tile_k + c);",
                         "uint32_t loc = (uint32_t)(c * tile_m + r);"),
    "no_padding": ("words += (cnt + 3) / 4 * 4;", "words += cnt;"),
    "tile_order_transposed": ("off[i * TK + j + 1] = (int32_t)words;",
                              "off[j * TM + i + 1] = (int32_t)words;"),
    "sign_dropped": ("return sign ? -v : v;", "return v;"),
    "exponent_bias_off_by_one": ("ldexp((double)(1024 + m), e - 25)", "ldexp((double)(1024 + m), e - 24)"),
    "truncating_fp16_rounding": ("double q = rint(ldexp(a, 10 - e));", "double q = floor(ldexp(a, 10 - e));"),
    "dropped_last_word": ("for (int64_t w = jb->off[t]; w < jb->off[t + 1]; ++w) {",
                          "for (int64_t w = jb->off[t]; w < jb->off[t + 1] - 1; ++w) {"),
    "transposed_B": ("bk[n] = ref_half_to_double(jb->B[n * jb->K + k]);",
                     "bk[n] = ref_half_to_double(jb->B[k * jb->N + n]);"),
    "decode_row_from_wrong_field": ("int64_t r = loc / tile_k, c = loc % tile_k;\n            int64_t gr",
                                    "int64_t r = loc % tile_k, c = loc / tile_k;\n            int64_t gr"),
    "v2_ties_to_higher_bank": ("if (ra > rb || (ra == rb && a < b)) break;",
                               "if (ra > rb || (ra == rb && a > b)) break;"),
    "v2_fewest_first": ("if (ra > rb || (ra == rb && a < b)) break;", "if (ra < rb || (ra == rb && a < b)) break;"),
    "v2_unswizzled_bank": ("uint32_t off = x ^ ((x >> 3) & 0x70u);\n    return (off >> 2) & 31u;",
                           "uint32_t off = x;\n    return (off >> 2) & 31u;"),
    "sentinel_not_skipped_in_spmm": ("if (loc == 0xFFFF) continue;\n                int64_t r = loc / jb->tile_k",
                                     "if (loc == 0xFFFE) continue;\n                int64_t r = loc / jb->tile_k"),
}


def _pin_suite():
    g = pins.GOLDEN["examples"]
    yield lambda: [pins.test_golden_encode(e) for e in g]
    yield lambda: [pins.test_golden_decode(e) for e in g]
    yield pins.test_golden_spmm
    yield lambda: pins.test_round_trip_and_invariants((200, 136, 64, 64), 0.2)
    yield lambda: pins.test_spmm_equals_dense_bruteforce(130, 200, 16, 64, 64, 0.3)
    yield pins.test_half_to_double_all_patterns
    yield pins.test_double_to_half_matches_numpy
    yield pins.test_permutation_is_exact_product
    yield lambda: [pins_v2.test_golden_orders(c) for c in pins_v2.GOLDEN["cases"]]
    yield lambda: pins_v2.test_v2_is_a_reordering_with_the_rule_properties(80, "uniform")


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    src = SRC.read_text()
    assert src.count(old) == 1, f"mutation anchor for {name} not unique"
    (tmp_path / "m.c").write_text(src.replace(old, new))
    so = tmp_path / "m.so"
    subprocess.check_call(["gcc", "-O2", "-ffp-contract=off", "-std=c11", "-shared", "-fPIC",
                           "-pthread", str(tmp_path / "m.c"), "-o", str(so), "-lm"])
    monkeypatch.setattr(oracle, "_lib", oracle.configure(ctypes.CDLL(str(so))))
    failures = 0
    for pin in _pin_suite():
        try:
            with np.errstate(all="ignore"):
                pin()
        except (AssertionError, oracle.OracleError):
            failures += 1
    assert failures > 0, f"no pin caught mutant {name}"
