"""Planted mistakes: each mutant is a copy of the oracle's C source with one
plausible error (a wrong rounding rule, a transposed operand, a dropped term,
a wrong index or constant), built on the CPU into a temporary directory.  The
pins of the other test files must reject every mutant, and accept the
unmodified copy."""
import importlib.util
import json
import os
import shutil
import sys

import numpy as np
import pytest

import test_oracle_codecs as C
import test_oracle_gemm as G
import test_oracle_quant as Q

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

ROW_CASES = json.load(open(os.path.join(Q.GOLD, "quantize_rows.json")))["cases"]
Q80_CASES = Q.Q80["cases"]

PINS = [
    C.test_bf16_encode_closed_form, C.test_bf16_decode_exhaustive, C.test_f16_decode_exhaustive,
    C.test_e4m3_decode_table, C.test_e4m3_saturation_closed_form, C.test_e4m3_all_bf16_values,
    lambda o: C.test_f16_encode_vs_numpy(o),
    *[(lambda c: (lambda o: Q.test_quantize_rows_golden(o, c)))(c) for c in ROW_CASES],
    lambda o: Q.test_quantize_rows_absmax_invariant(o, 0),
    lambda o: Q.test_quantize_rows_absmax_invariant(o, 1),
    lambda o: Q.test_quantize_weight_tensor(o, 0),
    Q.test_quantize_weight_axis_is_rowwise,
    *[(lambda c: (lambda o: Q.test_q8_0_golden_blocks(o, c)))(c) for c in Q80_CASES],
    Q.test_q8_0_invariants, Q.test_q8_0_short_tail, Q.test_q8_0_grid_roundtrip,
    Q.test_requant_same_scale_rows_are_unchanged, Q.test_requant_invariants,
    Q.test_requant_e4m3_closed_form, Q.test_requant_e4m3_invariants,
    lambda o: Q.test_requant_equals_row_quantizer_on_bf16_exact_rows(o, 0),
    lambda o: Q.test_requant_equals_row_quantizer_on_bf16_exact_rows(o, 1),
    G.test_gemm_i8_bruteforce_tiny,
    lambda o: G.test_gemm_i8_vs_numpy_int64(o, 7, 9, 33),
    G.test_gemm_i8_int32_range_check, G.test_gemm_e4m3_vs_numpy,
    G.test_epilogue_closed_form, G.test_epilogue_axis_scale_indexes_columns,
    G.test_linear_fwd_reduces_to_integer_matmul, G.test_linear_dgrad_reduces_to_integer_matmul,
    G.test_lowrank_vs_numpy, G.test_svdq_zero_factors_is_float_linear,
    lambda o: G.test_svdq_zero_residual_is_lowrank_product(o, 0),
    lambda o: G.test_svdq_zero_residual_is_lowrank_product(o, 1),
    lambda o: G.test_dequant_e4m3_bf16_vs_torch(o, 3.1e-5), G.test_q8_0_dequantize_bf16_vs_torch,
    G.test_linear_bf16_vs_numpy_and_textbook, G.test_weight_only_forwards_compose,
    G.test_gelu_closed_forms_and_library, G.test_row_absmax_and_activated_forward,
]

# (name, text in oracle.c, replacement)
MUTANTS = [
    ("bf16 ties away", "if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;",
     "if (lo >= 0x8000u) hi += 1u;"),
    ("bf16 truncation", "if (lo > 0x8000u || (lo == 0x8000u && (hi & 1u))) hi += 1u;", ""),
    ("f16 exponent bias", "(uint16_t)((E + 15) << 10)", "(uint16_t)((E + 16) << 10)"),
    ("f16 decode subnormal step", "v = ldexp((double)m, -24)", "v = ldexp((double)m, -23)"),
    ("e4m3 exponent bias", "(uint8_t)((E + 7) << 3)", "(uint8_t)((E + 8) << 3)"),
    ("e4m3 mantissa truncated", "double m = nearbyint((ldexp(a, -E) - 1.0) * 8.0);",
     "double m = floor((ldexp(a, -E) - 1.0) * 8.0);"),
    ("e4m3 saturates to NaN", "return (uint8_t)(sign | 0x7Eu);", "return (uint8_t)(sign | 0x7Fu);"),
    ("int8 ties away", "float r = nearbyintf(v);", "float r = roundf(v);"),
    ("int8 truncation", "float r = nearbyintf(v);", "float r = truncf(v);"),
    ("scale by reciprocal", "return (a < 1e-10f) ? 1e-10f : a / qmax_of(qt);",
     "return (a < 1e-10f) ? 1e-10f : a * (1.0f / qmax_of(qt));"),
    ("no scale floor", "return (a < 1e-10f) ? 1e-10f : a / qmax_of(qt);",
     "return (a <= 0.0f) ? 1.0f : a / qmax_of(qt);"),
    ("e4m3 qmax 127", "return qt == ORC_E4M3 ? 448.0f : 127.0f;", "return 127.0f;"),
    ("row absmax skips last column", "for (int64_t k = 0; k < K; ++k) {\n      float v = fabsf(orc_bf16_to_f32(row[k]));",
     "for (int64_t k = 0; k < K - 1; ++k) {\n      float v = fabsf(orc_bf16_to_f32(row[k]));"),
    ("tensor scale from first row", "for (int64_t i = 0; i < N * K; ++i) {\n    float v = fabsf",
     "for (int64_t i = 0; i < K; ++i) {\n    float v = fabsf"),
    ("q8_0 ties to even", "float r = roundf(x[start + j] / scale);", "float r = nearbyintf(x[start + j] / scale);"),
    ("q8_0 scale big-endian", "blk[0] = (uint8_t)(d & 0xFF);          /* little-endian f16 */\n    blk[1] = (uint8_t)(d >> 8);",
     "blk[1] = (uint8_t)(d & 0xFF);\n    blk[0] = (uint8_t)(d >> 8);"),
    ("q8_0 floor 0", "float scale = (max_abs < 1e-10f) ? 1e-10f : max_abs / 127.0f;",
     "float scale = (max_abs <= 0.0f) ? 1.0f : max_abs / 127.0f;"),
    ("q8_0 block stride 32", "const uint8_t* blk = blocks + (i / Q80_BLOCK) * Q80_BYTES;",
     "const uint8_t* blk = blocks + (i / Q80_BLOCK) * Q80_BLOCK;"),
    ("q8_0 code offset", "y[i] = block_scale_f16(blk) * (float)(int8_t)blk[2 + i % Q80_BLOCK];",
     "y[i] = block_scale_f16(blk) * (float)(int8_t)blk[1 + i % Q80_BLOCK];"),
    ("requant qmax 128", "float sn = absmax_scale(a, qt);", "float sn = a / 128.0f;"),
    ("requant e4m3 scale by 127", "float sn = absmax_scale(a, qt);", "float sn = absmax_scale(a, ORC_INT8);"),
    ("requant e4m3 int8 codes", "q[n * K + k] = encode_code(deq[k] / sn, qt);",
     "q[n * K + k] = encode_code(deq[k] / sn, ORC_INT8);"),
    ("requant row stride", "orc_q8_0_dequantize(blocks + n * bpr * Q80_BYTES, K, deq);",
     "orc_q8_0_dequantize(blocks + n * K, K, deq);"),
    ("gemm nt transposed B", "sum += (int64_t)A[m * K + k] * (int64_t)B[n * K + k];",
     "sum += (int64_t)A[m * K + k] * (int64_t)B[k * N + n];"),
    ("gemm nn transposed B", "sum += (int64_t)A[m * N + n] * (int64_t)B[n * K + k];",
     "sum += (int64_t)A[m * N + n] * (int64_t)B[k * N + n];"),
    ("gemm no int32 check", "if (sum > INT32_MAX || sum < INT32_MIN) overflow = 1;\n      acc[m * N + n]",
     "acc[m * N + n]"),
    ("epilogue weight scale by row", "float u = t * s_w[w_axis ? n : 0];", "float u = t * s_w[w_axis ? m : 0];"),
    ("epilogue drops bias", "if (bias) u = u + orc_bf16_to_f32(bias[n]);", ""),
    ("epilogue drops row scale", "float t = (float)acc[m * N + n] * s_row[m];", "float t = (float)acc[m * N + n];"),
    ("fp64 epilogue drops weight scale", "double u = acc[m * N + n] * (double)s_row[m] * (double)s_w[w_axis ? n : 0];",
     "double u = acc[m * N + n] * (double)s_row[m];"),
    ("e4m3 gemm sign", "sum += p;\n        asum += fabs(p);\n      }\n      acc[m * N + n] = sum;",
     "sum += fabs(p);\n        asum += fabs(p);\n      }\n      acc[m * N + n] = sum;"),
    ("float8 dequant drops scale", "w[i] = orc_f32_to_bf16(orc_e4m3_to_f32(q[i]) * s);",
     "w[i] = orc_f32_to_bf16(orc_e4m3_to_f32(q[i]));"),
    ("gguf bf16 code offset", "w[i] = orc_f32_to_bf16(block_scale_f16(blk) * (float)(int8_t)blk[2 + i % Q80_BLOCK]);",
     "w[i] = orc_f32_to_bf16(block_scale_f16(blk) * (float)(int8_t)blk[1 + i % Q80_BLOCK]);"),
    ("bf16 linear transposed w", "(double)orc_bf16_to_f32(w[n * K + k]);", "(double)orc_bf16_to_f32(w[k * N + n]);"),
    ("bf16 linear drops bias", "if (bias) v = v + orc_bf16_to_f32(bias[n]);", ""),
    ("gelu scaled argument", "r = 0.5 * x * (1.0 + erf(x / sqrt(2.0)));", "r = 0.5 * x * (1.0 + erf(x / 2.0));"),
    ("gelu tanh cubic dropped", "(x + 0.044715 * x * x * x)", "(x)"),
    ("row absmax skips the last column", "for (int64_t n = 0; n < N; ++n) {\n      float v = fabsf(orc_bf16_to_f32(y[m * N + n]));",
     "for (int64_t n = 0; n + 1 < N; ++n) {\n      float v = fabsf(orc_bf16_to_f32(y[m * N + n]));"),
    ("lowrank L1 transposed", "(double)orc_bf16_to_f32(l1[k * r + j])", "(double)orc_bf16_to_f32(l1[j * K + k])"),
    ("lowrank up drops a term", "for (int64_t j = 0; j < r; ++j) {\n        double p", "for (int64_t j = 1; j < r; ++j) {\n        double p"),
]


def _load_copy(tmp, tag, old=None, new=None):
    pkg = os.path.join(tmp, "orcmut_%s" % tag)
    os.makedirs(pkg, exist_ok=True)
    for f in ("__init__.py", "oracle.h", "svdquant.py"):
        shutil.copy(os.path.join(ORACLE_DIR, f), pkg)
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    if old is not None:
        assert src.count(old) >= 1, "mutation site not found: %r" % old
        src = src.replace(old, new, 1)
    open(os.path.join(pkg, "oracle.c"), "w").write(src)
    name = "orcmut_%s" % tag
    spec = importlib.util.spec_from_file_location(name, os.path.join(pkg, "__init__.py"),
                                                  submodule_search_locations=[pkg])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _failures(mod):
    bad = 0
    for pin in PINS:
        try:
            with np.errstate(all="ignore"):
                pin(mod)
        except (AssertionError, OverflowError, ValueError, IndexError, pytest.fail.Exception):
            bad += 1
    return bad


def test_unmodified_copy_passes_every_pin(tmp_path):
    assert _failures(_load_copy(str(tmp_path), "clean")) == 0


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_rejected(tmp_path, name, old, new):
    tag = "m%d" % MUTANTS.index((name, old, new))
    assert _failures(_load_copy(str(tmp_path), tag, old, new)) >= 1, name
