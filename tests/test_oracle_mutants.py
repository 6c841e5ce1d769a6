"""The pins must catch plausible oracle mistakes.  Each case copies the oracle
source into a temporary directory, plants one mistake there (a wrong tie rule,
a dropped term, a wrong bias, a transposed operand, a lost sign ...), builds
that copy, and checks that at least one pin from the other oracle test
modules fails against it.  Nothing here touches the real oracle build."""
import ctypes
import os
import shutil
import subprocess

import pytest

import oracle
from tests import test_oracle_formats as F
from tests import test_oracle_gemm as G
from tests import test_oracle_quant as Q
from tests import test_oracle_quotient as D
from tests import test_oracle_static_concat as S

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "ties_away_from_even": ("pick = (c % 2 == 0) ? c : c + 1;", "pick = c + 1;"),
    "mx_bias_off_by_one": ("ceil(log2(amax / 448.0)) + 127.0", "ceil(log2(amax / 448.0)) + 126.0"),
    "mx_floor_not_ceil": ("ceil(log2(amax / 448.0))", "floor(log2(amax / 448.0))"),
    "rowwise_wrong_divisor": ("float s = (amax == 0.0f) ? 1.0f : (float)((double)amax / 448.0);",
                              "float s = (amax == 0.0f) ? 1.0f : (float)((double)amax / 480.0);"),
    "tensor_scale_wrong_divisor": ("return (amax == 0.0f) ? 1.0f : (float)((double)amax / 448.0);",
                                   "return (amax == 0.0f) ? 1.0f : (float)((double)amax / 480.0);"),
    "static_scale_multiplied": ("bf16_to_float(c->x[r * c->ld_x + j]) / c->s;",
                                "bf16_to_float(c->x[r * c->ld_x + j]) * c->s;"),
    "sign_dropped": ("signbit(v) ? 0x80 : 0x00", "0x00"),
    "overflow_to_nan": ("if (a >= 448.0) return sign | 0x7E;", "if (a >= 448.0) return sign | 0x7F;"),
    "b_scale_dropped": ("(double)g->sa[i] * (double)g->sb[j]", "(double)g->sa[i]"),
    "b_transposed": ("double prod = g->dec[a[t]] * g->dec[b[t]];",
                     "double prod = g->dec[a[t]] * g->dec[g->qb[(t * g->n + j) % (g->n * g->k)]];"),
    "mx_block_index_dropped": ("(int)g->sfb[j * nkb + blk] - 254", "(int)g->sfb[j * nkb] - 254"),
    "subnormal_decode_wrong": ("mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    "rowwise_reciprocal_multiply": ("float v = bf16_to_float(xr[j]) / s;",
                                    "float v = bf16_to_float(xr[j]) * (1.0f / s);"),
    "static_reciprocal_multiply": ("float v = bf16_to_float(c->x[r * c->ld_x + j]) / c->s;",
                                   "float v = bf16_to_float(c->x[r * c->ld_x + j]) * (1.0f / c->s);"),
}

PINS = [
    F.test_decode_matches_bitfield_definition, F.test_decode_invariants,
    F.test_encode_midpoints_go_to_even_code, F.test_encode_round_trip_and_saturation,
    F.test_mx_exponent_special_values, F.test_mx_exponent_integer_closed_form,
    Q.test_rowwise_special_rows, Q.test_rowwise_invariants_random, Q.test_mx_special_blocks,
    G.test_all_ones_closed_form, G.test_selection_matrix_reproduces_rows_of_b,
    lambda o: G.test_mx_exact_against_integer_brute_force(o, 3, 4, 64),
    lambda o: G.test_rowwise_exact_against_integer_brute_force(o, 3, 5, 16),
    lambda o: S.test_tensor_scale_is_the_largest_row_scale(),
    lambda o: S.test_tensor_scale_closed_forms(3),
    lambda o: S.test_static_with_power_of_two_scale_is_exact_scaling(-1),
    lambda o: S.test_static_with_the_row_scale_is_the_row_quantizer(),
    D.test_rowwise_quotient_is_ieee_division_at_ties, D.test_rowwise_quotient_is_ieee_division_many_scales,
    D.test_static_quotient_is_ieee_division,
]


def _build_mutant(tmp_path, before, after):
    src = open(SRC).read()
    assert src.count(before) == 1, before
    d = tmp_path / "mut"
    d.mkdir()
    shutil.copy(os.path.join(os.path.dirname(SRC), "oracle.h"), d / "oracle.h")
    (d / "oracle.c").write_text(src.replace(before, after))
    out = d / "liboracle_mut.so"
    subprocess.run(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", "-fno-fast-math",
                    "-ffp-contract=off", "-o", str(out), str(d / "oracle.c"), "-lm"], check=True)
    return str(out)


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, monkeypatch, orc, name):
    before, after = MUTANTS[name]
    path = _build_mutant(tmp_path, before, after)
    real = oracle.lib()
    mut = ctypes.CDLL(path)
    for fn in ("orc_e4m3_decode", "orc_e4m3_encode", "orc_mx_exponent", "orc_quantize_rowwise",
               "orc_mx_quantize", "orc_gemm_rowwise", "orc_gemm_mx", "orc_tensor_scale", "orc_quantize_static"):
        getattr(mut, fn).argtypes = getattr(real, fn).argtypes
        getattr(mut, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", mut)
    caught = []
    for pin in PINS:
        try:
            pin(oracle)
        except AssertionError:
            caught.append(getattr(pin, "__name__", "lambda"))
    assert caught, f"no pin caught the planted mistake {name!r}"
