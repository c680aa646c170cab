"""Plant plausible mistakes in a copy of the oracle and check that the pins
catch every one of them.  The copies are built in a temporary directory on the
CPU; the oracle in the repository is never modified."""
import importlib.util
import os
import sys

import pytest

import oracle_pins

ORACLE_DIR = os.path.join(os.path.dirname(os.path.dirname(os.path.abspath(__file__))), "oracle")

# (name, text in qg_oracle.c, replacement): one planted mistake each
MUTANTS = [
    ("tie_to_odd_code", "(i % 2 == 0) ? i : i + 1", "(i % 2 == 0) ? i + 1 : i"),
    ("tie_rounds_down", "if (m == mid) return", "if (m == mid && 0) return"),
    ("sign_lost_on_negative_zero", "signbit(x) ? 8u : 0u", "(x < 0.0f) ? 8u : 0u"),
    ("no_saturation", "return (uint8_t)(sign | 7u);", "return (uint8_t)(sign | 0u);"),
    ("rank_off_by_one", "ceil(alpha * (double)n) - 1", "ceil(alpha * (double)n)"),
    ("rank_floor", "ceil(alpha * (double)n) - 1", "floor(alpha * (double)n) - 1"),
    ("delta_at_ties_too", "if (fabsf(a) > T) {\n                if (nnz >= cap)", "if (fabsf(a) >= T) {\n                if (nnz >= cap)"),
    ("clamp_drops_sign", "copysignf(T, a) : a;", "T : a;"),
    ("scale_inverted", "*s_out = amax / 6.0f;", "*s_out = 6.0f / amax;"),
    ("scale_not_max_based", "*r_out = r;", "*r_out = r * 0.5f;"),
    ("row_nibbles_swapped",
     "codes[i * (K / 2) + k / 2] =\n                (uint8_t)(orc_e2m1_encode(x0) | (orc_e2m1_encode(x1) << 4));",
     "codes[i * (K / 2) + k / 2] =\n                (uint8_t)(orc_e2m1_encode(x1) | (orc_e2m1_encode(x0) << 4));"),
    ("col_amax_first_row_only",
     "for (int64_t k = 0; k < K; ++k)\n            if (fabsf(W[k * N + j]) > amax)",
     "for (int64_t k = 0; k < 1; ++k)\n            if (fabsf(W[k * N + j]) > amax)"),
    ("gemm_nibbles_swapped",
     "wt[j * K + k] = orc_e2m1_value((k & 1) ? (uint8_t)(b >> 4) : (uint8_t)(b & 15u));",
     "wt[j * K + k] = orc_e2m1_value((k & 1) ? (uint8_t)(b & 15u) : (uint8_t)(b >> 4));"),
    ("gemm_drops_last_k", "for (int64_t k = 0; k < K; ++k) sum +=",
     "for (int64_t k = 0; k < K - 1; ++k) sum +="),
    ("y_without_correction", "for (int64_t j = 0; j < N; ++j) y[j] += val[p] * (double)w[j];",
     "for (int64_t j = 0; j < N; ++j) y[j] += 0.0 * val[p] * (double)w[j];"),
    ("y_row_scale_twice", "acc[r * N + j] * (double)sA[i] * (double)sW[j]",
     "acc[r * N + j] * (double)sA[i] * (double)sA[i]"),
    ("spmm_wrong_row_of_w", "const float* w = W + (int64_t)col[p] * N;\n            for (int64_t j = 0; j < N; ++j) c[j]",
     "const float* w = W + (int64_t)(col[p] > 0 ? col[p] - 1 : 0) * N;\n            for (int64_t j = 0; j < N; ++j) c[j]"),
    ("delta_in_single", "val[nnz] = (double)a - (double)ac;", "val[nnz] = (double)(float)(a * 1.0000001f - ac);"),
    ("bits_packed_nibbles_swapped", "packed[j] = (uint8_t)(c0 | (c1 << 4));",
     "packed[j] = (uint8_t)(c1 | (c0 << 4));"),
    ("bits_packed_start_off_by_one", "uint32_t b0 = start + (uint32_t)(2 * j), b1 = b0 + 1u;",
     "uint32_t b0 = start + (uint32_t)(2 * j) + 1u, b1 = b0 + 1u;"),
    ("bits_packed_nan_keeps_sign", "uint8_t c0 = isnan(x0) ? 0u : orc_e2m1_encode(x0);",
     "uint8_t c0 = isnan(x0) ? (uint8_t)(signbit(x0) ? 8u : 0u) : orc_e2m1_encode(x0);"),
    ("mx_exponent_floor_rule", "ldexp(6.0, e) < (double)amax", "ldexp(8.0, e) <= (double)amax"),
    ("mx_exponent_not_minimal", "while (e < 127 && ldexp(6.0, e) < (double)amax) ++e;",
     "while (e < 127 && ldexp(6.0, e) < (double)amax) ++e;\n    if (amax > 0.0f && e < 127) ++e;"),
    ("mx_block_of_16", "mx_block(A + i * K + 32 * b, 1, 32, q)",
     "mx_block(A + i * K + 32 * b, 1, 16, q); mx_block(A + i * K + 32 * b + 16, 1, 16, q + 16)"),
    ("mx_gemm_scale_difference", "((int)sA[i * nb + b] - 127) + ((int)sW[j * nb + b] - 127)",
     "((int)sA[i * nb + b] - 127) - ((int)sW[j * nb + b] - 127)"),
    ("mx_cols_reads_transposed", "mx_block(W + 32 * b * N + j, N, 32, q)",
     "mx_block(W + 32 * b + j * K, 1, 32, q)"),
]


def _build_variant(tmp_path, name, find, repl, target="qg_oracle.c"):
    pkg = tmp_path / f"orc_{name}"
    pkg.mkdir()
    for fname in ("qg_oracle.c", "__init__.py"):
        src = open(os.path.join(ORACLE_DIR, fname)).read()
        if fname == target:
            assert src.count(find) >= 1, f"mutation anchor not found: {name}"
            src = src.replace(find, repl, 1)
        (pkg / fname).write_text(src)
    modname = f"orc_mutant_{name}"
    spec = importlib.util.spec_from_file_location(modname, pkg / "__init__.py",
                                                  submodule_search_locations=[str(pkg)])
    mod = importlib.util.module_from_spec(spec)
    sys.modules[modname] = mod
    spec.loader.exec_module(mod)
    return mod


# the same, planted in the Python compositions of the gradient GEMMs
PY_MUTANTS = [
    ("dgrad_row_scale_dropped", "return scaled_product(acc, sd if rows is None",
     "return scaled_product(acc, 1.0 + 0 * sd if rows is None"),
    ("dgrad_weight_scale_of_dy", "cw, sw = quantize_rows(W)",
     "cw, sw = quantize_rows(W)\n    sw = sw * 0 + sd.max()"),
    ("wgrad_contraction_halved", "M = 2 * ca.shape[1]", "M = ca.shape[1]"),
    ("wgrad_dy_per_row", "cd, sd = quantize_cols(dY)",
     "cd, sd = quantize_cols(dY)\n    sd = sd * 0 + quantize_rows(dY)[1].max()"),
]


@pytest.mark.parametrize("name,find,repl,target",
                         [m + ("qg_oracle.c",) for m in MUTANTS]
                         + [m + ("__init__.py",) for m in PY_MUTANTS],
                         ids=[m[0] for m in MUTANTS + PY_MUTANTS])
def test_planted_mistake_is_caught(tmp_path, name, find, repl, target):
    mod = _build_variant(tmp_path, name, find, repl, target)
    caught = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(mod)
        except AssertionError:
            caught.append(pin.__name__)
            break
    assert caught, f"no pin catches the planted mistake '{name}'"
