"""Plant one plausible mistake at a time in a copy of the oracle's C source
(on the CPU, in a temporary directory) and require the pins to catch it.

This shows that the pins constrain every step of the oracle: a dropped term,
a wrong order, sign, index, constant or rounding rule fails at least one.
"""
import os

import pytest

import oracle
import oracle_pins

# (name, text in rrf_oracle.c, replacement)
MUTANTS = [
    ("sum starts from +0",
     "float acc = oracle_bf16_to_float(x[0][k]);\n    for (int r = 1; r < R; ++r)",
     "float acc = 0.0f;\n    for (int r = 0; r < R; ++r)"),
    ("last input dropped", "for (int r = 1; r < R; ++r)", "for (int r = 1; r < R - 1; ++r)"),
    ("float64 accumulator", "float acc = oracle_bf16_to_float(x[0][k]);",
     "double acc = oracle_bf16_to_float(x[0][k]);"),
    ("reversed rank order",
     "for (int r = 1; r < R; ++r) acc = acc + oracle_bf16_to_float(x[r][k]);",
     "for (int r = R - 1; r >= 1; --r) acc = acc + oracle_bf16_to_float(x[r][k]);"),
    ("residual not added",
     "float t = oracle_bf16_to_float(s) + oracle_bf16_to_float(res_in[base + j]);",
     "float t = oracle_bf16_to_float(s);"),
    ("eps outside the square root", "1.0f / sqrtf(ms + eps)", "1.0f / (sqrtf(ms) + eps)"),
    ("mean over cols - 1", "(float)ss / (float)cols", "(float)ss / (float)(cols - 1)"),
    ("weight offset dropped", "oracle_bf16_to_float(gamma[j]) + weight_offset;",
     "oracle_bf16_to_float(gamma[j]);"),
    ("weight offset subtracted", "oracle_bf16_to_float(gamma[j]) + weight_offset;",
     "oracle_bf16_to_float(gamma[j]) - weight_offset;"),
    ("no scale_ub clamp", "fminf(amax, scale_ub)", "amax"),
    ("no scale floor", "fmaxf(fminf(amax, scale_ub), SCALE_FLOOR)", "fminf(amax, scale_ub)"),
    ("e4m3fnuz maximum 240", "/ 448.0f", "/ 240.0f"),
    ("scale applied as a multiplier", "float v = y / scale;", "float v = y * scale;"),
    ("amax over h instead of y", "float ay = fabsf(y);", "float ay = fabsf(h);"),
    ("row stride lost", "const int64_t base = i * cols;", "const int64_t base = i;"),
    ("transposed sum index", "out[i * cols + j] = sum_element(x, R, i * cols + j);",
     "out[i * cols + j] = sum_element(x, R, j * rows + i);"),
    ("e4m3 ties away from zero", "(d == best_d && (c & 1) == 0)", "(d == best_d)"),
    ("e4m3 loses the sign of zero", "uint8_t sign = signbit(v) ? 0x80 : 0x00;",
     "uint8_t sign = (v < 0) ? 0x80 : 0x00;"),
    ("e4m3 overflow to NaN", "if (a > E4M3_MAX) return (uint8_t)(sign | 0x7E);",
     "if (a > E4M3_MAX) return 0x7F;"),
    ("e4m3 exponent bias off by one", "ldexp((double)(8 + m), e - 10)",
     "ldexp((double)(8 + m), e - 11)"),
    ("bf16 ties away from zero", "return (lo & 1) ? hi : lo;", "return hi;"),
    ("bf16 truncation", "if (dhi < dlo) return hi;", "if (0) return hi;"),
    ("GEMM last k dropped", "for (int64_t k = 0; k < K; ++k)\n                S +=",
     "for (int64_t k = 0; k < K - 1; ++k)\n                S +="),
    ("GEMM b read transposed", "oracle_e4m3_decode(b[n * K + k])",
     "oracle_e4m3_decode(b[(k * N + n) % (N * K)])"),
    ("GEMM one scale for all rows", "S * (double)a_scale[m] * (double)b_scale[n]",
     "S * (double)a_scale[0] * (double)b_scale[n]"),
    ("GEMM bias dropped", "if (bias != NULL) y += (double)oracle_bf16_to_float(bias[n]);", ""),
    ("GEMM rounds through fp32", "out[m * N + n] = oracle_bf16_round_double(y);",
     "out[m * N + n] = oracle_bf16_round((float)y);"),
    ("double rounding ties up", "pick = (fmod(k, 2.0) == 0.0) ? lo : hi;", "pick = hi;"),
    ("double rounding truncates", "else if (hi - a < a - lo) pick = hi;", "else if (0) pick = hi;"),
    ("double rounding 7 significant bits", "int q_exp = e - 8;", "int q_exp = e - 7;"),
    ("MX scale rounded up", "int c = (e - 1) - 8 + 127;", "int c = e - 8 + 127;"),
    ("MX e4m3 exponent 7", "int c = (e - 1) - 8 + 127;", "int c = (e - 1) - 7 + 127;"),
    ("MX amax over half a block", "if (fabsf(y[k]) > amax) amax = fabsf(y[k]);",
     "if (k < 16 && fabsf(y[k]) > amax) amax = fabsf(y[k]);"),
    ("MX zero block scale 1", "if (!(amax > 0.0f)) return 0;", "if (!(amax > 0.0f)) return 127;"),
    ("MX scale applied as a multiplier", "float v = y[k] * inv_x;", "float v = y[k] / inv_x;"),
    ("MX GEMM block shifted", "sa[m * nb + k / MX_BLOCK]", "sa[m * nb + (k / MX_BLOCK + 1) % nb]"),
    ("MX GEMM b scaled by a's row", "sb[n * nb + k / MX_BLOCK]", "sb[(m % N) * nb + k / MX_BLOCK]"),
    ("E8M0 bias 126", "return ldexp(1.0, (int)c - 127);", "return ldexp(1.0, (int)c - 126);"),
    ("MX GEMM bias dropped", "if (bias != NULL) S += (double)oracle_bf16_to_float(bias[n]);", ""),
]


def _build_mutant(tmp_path, old, new):
    with open(os.path.join(os.path.dirname(oracle.__file__), "rrf_oracle.c")) as fh:
        src = fh.read()
    assert src.count(old) >= 1, f"mutation site not found: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    return oracle.Oracle(oracle.build(force=True, src=str(path), out=str(tmp_path / "m.so")))


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    mutant = _build_mutant(tmp_path, old, new)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mutant)
        except (AssertionError, ValueError, FloatingPointError):
            caught.append(pin.__name__)
    assert caught, f"no pin caught the mutant '{name}'"
