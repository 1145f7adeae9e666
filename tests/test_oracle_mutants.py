"""Every plausible mistake planted in the C oracle must fail at least one pin.

Each mutant is a one-spot edit of ``oracle/lcla_oracle.c`` (a dropped term, a
wrong sign or index, a transposed operand, a shifted block boundary ...),
compiled on the CPU into a temporary directory and run against every pin.
"""
import os

import pytest

import oracle
from pins import ALL_PINS

ROT_OK = """        y[2 * p] = a * (double)c[p] - b * (double)s[p];
        y[2 * p + 1] = a * (double)s[p] + b * (double)c[p];"""

MUTANTS = {
    # rotary embedding
    "rotation_not_orthogonal": [(ROT_OK, ROT_OK.replace("- b * (double)s[p]", "+ b * (double)s[p]", 1))],
    "rotation_reversed": [(ROT_OK, """        y[2 * p] = a * (double)c[p] + b * (double)s[p];
        y[2 * p + 1] = -a * (double)s[p] + b * (double)c[p];""")],
    "rotation_half_split_pairs": [("        double a = x[2 * p], b = x[2 * p + 1];",
                                   "        double a = x[p], b = x[p + d / 2];")],
    "rotation_uses_row_zero": [("    const float *c = cs + (size_t)n * (d / 2);",
                                "    const float *c = cs;")],
    # feature map
    "relu_dropped": [("return x < 0.0 ? 0.0 : x;", "return x;")],
    "relu_is_abs": [("return x < 0.0 ? 0.0 : x;", "return x < 0.0 ? -x : x;")],
    "bf16_widening_shift": [("[i]) << 16;", "[i]) << 15;")],
    # masked (pair-by-pair) route
    "masked_rotated_denominator": [("den += dot(kf + (size_t)j * d, qf, d);",
                                    "den += dot(kr + (size_t)j * d, qr, d);")],
    "masked_exclusive_block": [("long last = ((long)(i / block_len) + 1) * (long)block_len;",
                                "long last = ((long)(i / block_len)) * (long)block_len;")],
    "masked_token_causal_inside_block": [("long last = ((long)(i / block_len) + 1) * (long)block_len;",
                                          "long last = i + 1;")],
    "masked_eps_doubled": [("o[c] = num[c] / (den + eps);", "o[c] = num[c] / (den + 2 * eps);")],
    "masked_value_of_query_token": [("                    load_row(v, dtype, N, H, d, b, j, h, vj);\n"
                                     "                    for (int c = 0; c < d; ++c) num[c] += vj[c] * a;",
                                     "                    load_row(v, dtype, N, H, d, b, i, h, vj);\n"
                                     "                    for (int c = 0; c < d; ++c) num[c] += vj[c] * a;")],
    # recurrence route
    "recurrence_transposed_state": [("acc[(size_t)c * d + e] += vj[c] * kr[e];",
                                     "acc[(size_t)e * d + c] += vj[c] * kr[e];")],
    "recurrence_rotated_key_sum": [("acc[(size_t)d * d + e] += kf[e];", "acc[(size_t)d * d + e] += kr[e];")],
    "recurrence_dropped_eps": [("double den = dot(P + (size_t)d * d, qf, d) + eps;",
                                "double den = dot(P + (size_t)d * d, qf, d);")],
    "recurrence_exclusive_prefix": [("order[next].tok < j1;", "order[next].tok < j0;")],
    "recurrence_unrotated_query": [("    rotate(qf, cs, sn, i, d, qr);\n    double den = dot(P",
                                    "    rotate(qf, cs, sn, 0, d, qr);\n    double den = dot(P")],
    # row subsets (rows=): each requested row goes to its own slot, in token order
    "recurrence_rows_slot_is_visit_order": [
        ("out + (((size_t)b * nrows + (size_t)order[next].slot) * H + h)",
         "out + (((size_t)b * nrows + (size_t)next) * H + h)")],
    "recurrence_rows_not_sorted": [("    if (rows) qsort(order,", "    if (0) qsort(order,")],
    "masked_rows_ignored": [("long i = rows ? (long)rows[r] : (long)r;", "long i = (long)r;")],
    # step route
    "step_ignores_carried_state": [("S[x] += st[x];", "S[x] += 0.0 * st[x];")],
    "step_save_inverted": [("if (save) memcpy(st, S,", "if (!save) memcpy(st, S,")],
}


def _mutate(src, edits):
    for old, new in edits:
        assert src.count(old) == 1, f"mutation site not unique/present: {old!r}"
        src = src.replace(old, new)
    return src


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    src = open(oracle.SOURCE).read()
    path = tmp_path / f"{name}.c"
    path.write_text(_mutate(src, MUTANTS[name]))
    so = oracle.compile_source(str(path), str(tmp_path / f"lib{name}.so"))
    orc = oracle.Oracle(so)
    failures = []
    for pin in ALL_PINS:
        try:
            pin(orc)
        except (AssertionError, ValueError) as e:
            failures.append(pin.__name__)
    assert failures, f"mutant {name} passed every pin"


def test_unmutated_copy_passes(tmp_path):
    """Control: the same build path on the untouched source passes every pin."""
    path = tmp_path / "ok.c"
    path.write_text(open(oracle.SOURCE).read())
    orc = oracle.Oracle(oracle.compile_source(str(path), str(tmp_path / "libok.so")))
    for pin in ALL_PINS:
        pin(orc)
