"""The CPU oracle against its pins, and planted mistakes against the pins.

The oracle is the reference the CUDA path is compared with, so it is first tied
to facts outside itself (see ``oracle_pins``).  To show the pins have teeth,
``test_planted_mistake_is_caught`` compiles copies of ``oracle.c`` that each
carry one plausible mistake (wrong zero point, reversed bit order, wrong group
size, dropped permutation, off-by-one offsets, wrong rounding, ...) and checks
that at least one pin fails for every copy.  Mutants run in a subprocess so a
crash in one counts as caught without taking down the test run.
"""
import os
import subprocess
import sys
from concurrent.futures import ThreadPoolExecutor

import numpy as np
import pytest

import oracle
from tests import oracle_pins

HERE = os.path.dirname(os.path.abspath(__file__))


@pytest.mark.parametrize("pin", oracle_pins.PINS, ids=lambda p: p.__name__)
def test_pin(orc, pin):
    pin(orc)


# (name, text in oracle.c, replacement, which occurrence)
MUTANTS = [
    ("zero_point_dequant", "(double)(q - (1 << (b - 1))) * s;\n            }",
     "(double)(q - (1 << (b - 1)) + 1) * s;\n            }", 0),
    ("zero_point_gemm", "double w = (double)(q - (1 << (b - 1))) * s;",
     "double w = (double)(q - (1 << (b - 1)) - 1) * s;", 0),
    ("sign_gemm", "double w = (double)(q - (1 << (b - 1))) * s;",
     "double w = (double)((1 << (b - 1)) - q) * s;", 0),
    ("msb_first_read", "q |= ((word >> (p % 32)) & 1u) << t;",
     "q |= ((word >> (p % 32)) & 1u) << (b - 1 - t);", 0),
    ("msb_first_pack", "if ((q >> t) & 1u) qw", "if ((q >> (b - 1 - t)) & 1u) qw", 0),
    ("word_order_pack", "qw[(off + p / 32) * N + n] |= 1u << (p % 32);",
     "qw[(off + (b - 1) - p / 32) * N + n] |= 1u << (p % 32);", 0),
    ("group_size_64", "#define ORC_GROUP 128", "#define ORC_GROUP 64", 0),
    ("scale_group0_gemm", "J->scales[(int64_t)(k / ORC_GROUP) * J->N + n]", "J->scales[n]", 0),
    ("perm_dropped", "J->x[(int64_t)m * J->K + src]", "J->x[(int64_t)m * J->K + k]", 0),
    ("x_row_stride", "J->x[(int64_t)m * J->K + src]", "J->x[(int64_t)m + src]", 0),
    ("offset_shift", "{ off[j] = s; s += bits[j]; }", "{ s += bits[j]; off[j] = s - 2; if (off[j] < 0) off[j] = 0; }", 0),
    ("last_block_dropped_gemm", "for (int j = 0; j < nb; ++j) {\n            int b = J->bits[j];",
     "for (int j = 0; j < nb - 1; ++j) {\n            int b = J->bits[j];", 0),
    ("half_subnormal_exp", "ldexp((double)m, -24)", "ldexp((double)m, -25)", 0),
    ("half_bias", "ldexp((double)(1024 + m), e - 25)", "ldexp((double)(1024 + m), e - 24)", 0),
    ("round_ties_away", "(rem == half && (q & 1))", "(rem == half)", 0),
    ("round_truncate", "if (rem > half || (rem == half && (q & 1))) ++q;", "", 0),
    ("round_subnormal_shift", "28 - e;", "29 - e;", 0),
    ("code_check_dropped", "if (q >> b) return ORC_ERR_CODE;", "", 0),
    ("stream_bit_stride", "int64_t p = (int64_t)r * b + t;                 /* stream bit */",
     "int64_t p = (int64_t)r * (b + 1) + t;", 0),
    # the quantiser
    ("q_zero_point", "int b = bits[k / ORC_BLOCK], z = 1 << (b - 1);",
     "int b = bits[k / ORC_BLOCK], z = (1 << (b - 1)) - 1;", 0),
    ("q_base_width", "float r = a / (float)(1 << (bits[k / ORC_BLOCK] - 1));",
     "float r = a / (float)(1 << bits[k / ORC_BLOCK]);", 0),
    ("q_no_sqrt", "rintf(sqrtf(qs[g] / qmax) * 16.0f)", "rintf((qs[g] / qmax) * 16.0f)", 0),
    ("q_qscale_levels", "rintf(sqrtf(qs[g] / qmax) * 16.0f)", "rintf(sqrtf(qs[g] / qmax) * 15.0f)", 0),
    ("q_round_away", "float t = rintf(x * inv);", "float t = roundf(x * inv);", 0),
    ("q_candidate_grid", "(float)(32 + i) / 96.0f", "(float)(33 + i) / 96.0f", 0),
    ("q_argmin_last_tie", "if (i == 0 || e < best_e) {", "if (i == 0 || e <= best_e) {", 0),
    ("q_clamp_high", "hi = (float)((1 << b) - 1 - z);", "hi = (float)((1 << b) - z);", 0),
    # the KV-cache quantiser
    ("kv_butterfly_sign", "a[i + st] = x - y;", "a[i + st] = y - x;", 0),
    ("kv_no_inverse_scale", "(double)(u[i] / (float)D)", "(double)(u[i])", 0),
    ("kv_scale_divisor", "(double)(amax / (float)(z - 1))", "(double)(amax / (float)z)", 0),
    ("kv_round_away", "float r = rintf(u[32 * g + i] * inv);", "float r = roundf(u[32 * g + i] * inv);", 0),
    ("kv_group_of_32", "float a = fabsf(u[32 * g + i]);", "float a = fabsf(u[i]);", 0),
    ("q_group_of_row", "int g = k / ORC_GROUP;\n        if (g != g_cur) {",
     "int g = k / ORC_BLOCK / 4 % 2;\n        if (g != g_cur) {", 0),
]


def _mutate(src, find, repl, occ):
    idx = -1
    for _ in range(occ + 1):
        idx = src.index(find, idx + 1)
    return src[:idx] + repl + src[idx + len(find):]


def test_mutant_edits_apply():
    src = oracle.source_text()
    for name, find, repl, occ in MUTANTS:
        assert src.count(find) > occ, f"mutant {name}: text not found in oracle.c"


def _run_mutant(args):
    name, find, repl, occ, tmpdir = args
    lib = os.path.join(tmpdir, f"mut_{name}.so")
    oracle.compile_variant(_mutate(oracle.source_text(), find, repl, occ), lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), lib],
                       capture_output=True, text=True, timeout=300)
    return name, r.returncode, r.stdout[-400:]


def test_planted_mistake_is_caught(tmp_path):
    jobs = [(n, f, r, o, str(tmp_path)) for n, f, r, o in MUTANTS]
    with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
        results = list(ex.map(_run_mutant, jobs))
    survivors = [name for name, rc, _ in results if rc == 0]
    assert not survivors, f"planted mistakes not caught by any pin: {survivors}"


def test_unmutated_copy_passes_in_subprocess(tmp_path):
    lib = os.path.join(str(tmp_path), "copy.so")
    oracle.compile_variant(oracle.source_text(), lib)
    r = subprocess.run([sys.executable, os.path.join(HERE, "oracle_pins.py"), lib],
                       capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout


def test_oracle_rejects_bad_shapes(orc):
    with pytest.raises(oracle.OracleError):
        orc.word_rows(np.array([4], np.uint8), 33)
    with pytest.raises(oracle.OracleError):
        orc.word_rows(np.array([7], np.uint8), 32)
    with pytest.raises(oracle.OracleError):
        orc.qgemm_f64(np.zeros((1, 32)), np.full(32, 40, np.int32), np.zeros((4, 1), np.uint32),
                      np.zeros((1, 1), np.uint16), np.array([4], np.uint8))


def test_oracle_threads(orc):
    rng = np.random.default_rng(12)
    bits = rng.choice(oracle_pins.BITS, size=6).astype(np.uint8)
    _, codes, s, x, perm = oracle_pins._rand_problem(rng, bits, 37, M=2)
    qw = orc.pack(codes, bits)
    y1, n1 = orc.qgemm_f64(x, perm, qw, s, bits, threads=1)
    y4, n4 = orc.qgemm_f64(x, perm, qw, s, bits, threads=4)
    assert n1 == 1 and n4 == 4
    assert np.array_equal(y1, y4)
