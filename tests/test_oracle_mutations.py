"""The oracle's pins catch plausible mistakes in the oracle.

Each case plants one mistake in a temporary copy of oracle/qnt_oracle.c (one
exact text replacement), compiles it with the oracle's own flags into a
temporary folder, loads it through a copy of oracle/oracle.py, and runs the
pins named for it: every one of them must fail.  The committed oracle passes
the same pins in test_oracle.py.  CPU only; the mistakes live in temporary
copies and never reach the library or the GPU.
"""
import importlib.util
import os
import shutil
import subprocess

import pytest

from tests import test_oracle as T

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE = os.path.join(ROOT, "oracle")

# name -> (text in qnt_oracle.c, replacement, pins that must fail as (test, kwargs))
MUTATIONS = {
    # AFPQ: negative codes scaled by s+ and positive codes by s-
    "afpq_scales_swapped": (
        "return v > 0.0 ? v * o_h2d(s1) : v * o_h2d(s2);",
        "return v > 0.0 ? v * o_h2d(s2) : v * o_h2d(s1);",
        [(T.test_dequant_one_fp4_afpq_razer_int8_by_hand, {}), (T.test_dequant_matrix_by_hand, {"fmt": 3})]),
    # RaZeR: the sign order of the special values reversed in the decode
    "razer_sv_sign_order": (
        "return (code == 8 ? RAZER_SV[z & 3] : o_e2m1(code)) * o_h2d(s1);",
        "return (code == 8 ? RAZER_SV[(z ^ 1) & 3] : o_e2m1(code)) * o_h2d(s1);",
        [(T.test_dequant_one_fp4_afpq_razer_int8_by_hand, {}), (T.test_dequant_matrix_by_hand, {"fmt": 4})]),
    # INT8: every row dequantized with the first row's scale
    "int8_first_row_scale": (
        "out[i] = o_dequant_one(fmt, codes[i], s1[n], 0, 0); continue;",
        "out[i] = o_dequant_one(fmt, codes[i], s1[0], 0, 0); continue;",
        [(T.test_dequant_matrix_by_hand, {"fmt": 5})]),
    # INT8: the code read as unsigned
    "int8_code_unsigned": (
        "case OF_INT8: return (double)(int8_t)code * o_h2d(s1);",
        "case OF_INT8: return (double)(uint8_t)code * o_h2d(s1);",
        [(T.test_dequant_one_fp4_afpq_razer_int8_by_hand, {}), (T.test_dequant_matrix_by_hand, {"fmt": 5})]),
    # INT4: the zero point added instead of subtracted in the decode
    "int4_zero_sign": (
        "case OF_INT4: return (double)(code - z) * o_h2d(s1);",
        "case OF_INT4: return (double)(code + z) * o_h2d(s1);",
        [(T.test_dequant_one_fp4_afpq_razer_int8_by_hand, {}), (T.test_dequant_matrix_by_hand, {"fmt": 1})]),
    # FP4: a wrong magnitude in the E2M1 table (6 -> 5)
    "e2m1_table_entry": (
        "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0};",
        "{0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 5.0};",
        [(T.test_e2m1_table_golden, {}), (T.test_dequant_one_fp4_afpq_razer_int8_by_hand, {})]),
    # INT4 / INT8: ties rounded half away from zero instead of half to even
    "round_half_away_from_zero": (
        "static float rne(float v) { return rintf(v); }",
        "static float rne(float v) { return roundf(v); }",
        [(T.test_int_ties_round_half_to_even, {})]),
    # RaZeR: the squared errors summed left to right instead of as a tree
    "razer_sse_sequential": (
        "for (int width = 1; width < n; width *= 2)\n"
        "    for (int i = 0; i + width < n; i += 2 * width) t[i] = t[i] + t[i + width];\n"
        "  return t[0];",
        "double acc = 0.0;\n  for (int i = 0; i < n; i++) acc += t[i];\n  return acc;",
        [(T.test_razer_selector_uses_tree_order_sum, {})]),
}


def _mutant(tmp_path, name, old, new):
    src = open(os.path.join(ORACLE, "qnt_oracle.c")).read()
    assert src.count(old) == 1, f"{name}: the text to replace must occur exactly once"
    d = tmp_path / name
    d.mkdir()
    (d / "qnt_oracle.c").write_text(src.replace(old, new))
    shutil.copy(os.path.join(ORACLE, "oracle.py"), d / "oracle.py")
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math", "-fopenmp", "-fPIC",
                           "-shared", "-o", str(d / "liboracle.so"), str(d / "qnt_oracle.c"), "-lm"])
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", str(d / "oracle.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_pins_catch_planted_mistake(tmp_path, name):
    old, new, pins = MUTATIONS[name]
    mut = _mutant(tmp_path, name, old, new)
    for pin, kw in pins:
        with pytest.raises(AssertionError):
            pin(mut, **kw)
