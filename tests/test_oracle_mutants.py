"""Plant plausible mistakes in copies of the oracle source, build each copy on the
CPU, and require that at least one pin fails for every mutant. This shows the pins
would catch a dropped term, a wrong sign or index, or a transposed operand."""
import os
import subprocess
import tempfile

import pytest

import oracle
import pins
from oracle import build_oracle

SRC = os.path.join(os.path.dirname(build_oracle.__file__), "macaq_oracle.c")

# (name, original text, mutated text): each original must occur exactly once.
MUTANTS = [
    ("butterfly_sign", "v[i + h] = a - b;", "v[i + h] = b - a;"),
    ("butterfly_dropped_term", "v[i] = a + b;", "v[i] = a;"),
    ("no_normalisation", "for (int i = 0; i < 32; ++i) v[i] = v[i] * c;", "(void)c;"),
    ("exponent_offset", "int e = E - 2;", "int e = E - 1;"),
    ("normal_exponent_bias", "E = biased - 127;", "E = biased - 126;"),
    ("zero_tie_rule", "if (a <= 0.25f)      idx = 0;", "if (a < 0.25f)       idx = 0;"),
    ("saturation_threshold", "else if (a <= 5.0f)  idx = 6;", "else if (a < 6.0f)   idx = 6;"),
    ("nibble_order", "codes16[j] = (uint8_t)(lo | (hi << 4));", "codes16[j] = (uint8_t)(hi | (lo << 4));"),
    ("sign_dropped", "return (uint8_t)(sign | idx);", "return (uint8_t)(idx);"),
    ("multiplier_ignored", "v[i] = oracle_bf16_to_f32(x[r * ld + k]) * mult[k];",
     "v[i] = oracle_bf16_to_f32(x[r * ld + k]);"),
    ("inv_s_not_inverted", "inv_s[k] = 1.0f / s[k];", "inv_s[k] = s[k];"),
    ("hadamard_sign", "return parity ? -1 : 1;", "return parity ? 1 : -1;"),
    ("scale_layout_rowgroup", "(r % 32) * 16 + ((r / 32) % 4) * 4 + (j % 4);",
     "(r % 32) * 16 + ((r / 32) % 4) * 8 + (j % 4);"),
    ("dequant_scale_bias", "int e = (int)scales[r * Kb + k / 32] - 127;",
     "int e = (int)scales[r * Kb + k / 32] - 126;"),
    ("dequant_nibble", "uint8_t code = (k & 1) ? (byte >> 4) : (byte & 0xF);",
     "uint8_t code = (k & 1) ? (byte & 0xF) : (byte >> 4);"),
    ("gemm_transposed_weight", "acc += adec[k] * wr[k];",
     "acc += adec[k] * wdec[(k % N) * K + n % K];"),
    ("decode_exponent_bias", "ldexp(1.0 + 0.5 * m, ex - 1)", "ldexp(1.0 + 0.5 * m, ex)"),
    ("transform_f64_index", "acc += x[r * K + k] * mult[k] * (double)oracle_hadamard_entry(i, j);",
     "acc += x[r * K + k] * mult[k] * (double)oracle_hadamard_entry(j, i & 15);"),
    ("hessian_diagonal_only", "for (int j = 0; j < 32; ++j) Hb[i * 32 + j] += (double)v[i] * (double)v[j];",
     "Hb[i * 32 + i] += (double)v[i] * (double)v[i];"),
    ("block_error_index", "for (int j = 0; j < 32; ++j) r += H[i * 32 + j] * d[j];",
     "for (int j = 0; j < 32; ++j) r += H[i * 32 + j] * d[i];"),
    ("error_at_exponent_sign", "d[2 * j] = (double)v[2 * j] - ldexp(oracle_e2m1_decode(lo), e);",
     "d[2 * j] = (double)v[2 * j] - ldexp(oracle_e2m1_decode(lo), -e);"),
    ("search_nibble_order", "codes16[j] = (uint8_t)((hi << 4) | lo);", "codes16[j] = (uint8_t)((lo << 4) | hi);"),
    ("search_ties_replace", "if (!have || err < best) {", "if (!have || err <= best) {"),
    ("search_no_lower_candidate", "int cand[3] = {e0, e0 + 1, e0 - 1};", "int cand[3] = {e0, e0 + 1, e0 + 1};"),
    ("flip_gain_sign", "double dE = b2 - c;", "double dE = b2 + c;"),
    ("flip_update_sign", "g[j] = fma(-bdelta, H[bk * K + j], g[j]);", "g[j] = fma(bdelta, H[bk * K + j], g[j]);"),
    ("flip_ties_accepted", "if (dE < best) {", "if (dE <= best) {"),
    ("flip_neighbour", "int ni = idx[k] + dir;", "int ni = idx[k] + 2 * dir;"),
    ("flip_error_sign", "e[k] = (double)wv[k] - ldexp(kFlipGrid[idx[k]], (int)scales_row[k / 32] - 127);",
     "e[k] = (double)wv[k] + ldexp(kFlipGrid[idx[k]], (int)scales_row[k / 32] - 127);"),
    ("hessian_full_diagonal", "for (int64_t j = 0; j < K; ++j) H[i * K + j] += (double)v[i] * (double)v[j];",
     "H[i * K + i] += (double)v[i] * (double)v[i];"),
]


def _build_mutant(tmp, name, old, new):
    src = open(SRC).read()
    assert src.count(old) == 1, (name, src.count(old))
    path_c = os.path.join(tmp, f"m_{name}.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    path_so = os.path.join(tmp, f"m_{name}.so")
    inc = os.path.dirname(SRC)
    subprocess.run(["gcc", *build_oracle.CFLAGS, "-I", inc, "-o", path_so, path_c, "-lm"],
                   check=True, capture_output=True)
    return path_so


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, old, new):
    with tempfile.TemporaryDirectory() as tmp:
        so = _build_mutant(tmp, name, old, new)
        caught = []
        with oracle.use_library(so):
            for pin in pins.ALL_PINS:
                try:
                    pin()
                except AssertionError:
                    caught.append(pin.__name__)
        assert caught, f"no pin catches mutant {name}"
