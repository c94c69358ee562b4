"""Plant plausible mistakes in a copy of the CPU oracle and check that a pin fails.

Each mutation edits the C source of a private copy (built under a temporary
directory), loads it as a separate module and runs the closed-form, library
and brute-force pins of ``test_oracle_pins`` against it.  A mutation that no
pin notices would mean the pins leave that part of the oracle unchecked.
Every mutation keeps its memory accesses in bounds.  Everything runs on the
CPU.
"""
import importlib.util
import os
import shutil
import sys

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

MUTATIONS = {
    "kurtosis_dropped_square": ("m4 = m4 + q * q;", "m4 = m4 + q;"),
    "kurtosis_biased_mean": ("double mu = s / (double)n;", "double mu = s / (double)(n + 1);"),
    "kurtosis_m2_not_squared": ("m4 / (m2 * m2)", "m4 / m2"),
    "split_not_strict": ("if (kappa[j] > tau)", "if (kappa[j] >= tau)"),
    "zero_point_sign": ("double zq = rint(-lo / S);", "double zq = rint(lo / S);"),
    "code_minus_zero": ("double c = rint(v[kk] / S) + z;", "double c = rint(v[kk] / S) - z;"),
    "scale_divisor": ("diff / 15.0", "diff / 16.0"),
    "fp16_truncates": ("double q = rint(ldexp(a, 10 - E));", "double q = floor(ldexp(a, 10 - E));"),
    "layout_word_stride": ("* 16 + word * 4 + j / 2;\n            uint8_t c",
                           "* 16 + word * 2 + j / 2;\n            uint8_t c"),
    "layout_scale_slot_reversed": ("pscales[((t * S + g / 8) * 32 + r) * 8 + g % 8] = scales[i * G + g];",
                                "pscales[((t * S + g / 8) * 32 + r) * 8 + 7 - g % 8] = scales[i * G + g];"),
    "outlier_gather_reversed": ("poutl[((t * O8 + o / 8) * 32 + r) * 8 + o % 8] = w[i * k + idx[o]];",
                                  "poutl[((t * O8 + o / 8) * 32 + r) * 8 + o % 8] = w[i * k + idx[n_o - 1 - o]];"),
    "gemm_zero_index": ("(double)zeros[i * G + kk / 32]) * S;\n                double xv",
                        "(double)zeros[i * G + kk % G]) * S;\n                double xv"),
    "gemm_dequant_sign": ("double wd = ((double)codes[i * k + kk] - (double)zeros",
                          "double wd = ((double)codes[i * k + kk] + (double)zeros"),
    "gemm_outlier_x_index": ("double xv = spectra_ref_bf16_to_double(xr[idx[t]]);",
                             "double xv = spectra_ref_bf16_to_double(xr[t]);"),
    "bf16_truncates": ("double q = rint(ldexp(a, 7 - E));", "double q = floor(ldexp(a, 7 - E));"),
    "bf16_subnormal_step": ("double q = rint(ldexp(a, 133));", "double q = rint(ldexp(a, 134));"),
    "embed_row_from_position": ("const int64_t row = ids[r];", "const int64_t row = r;"),
    "embed_group_of_column": ("const int64_t grp = row * ngroups + col / 32;",
                              "const int64_t grp = row * ngroups + col % ngroups;"),
    "embed_outlier_value_slot": ("dst[idx[t]] = spectra_ref_bf16_to_double(w[row * k + idx[t]]);",
                                 "dst[idx[t]] = spectra_ref_bf16_to_double(w[row * k + t]);"),
    "bulk_columns_skip_first": ("        bulk_idx[p++] = j;\n    }", "        if (j > 0) bulk_idx[p++] = j;\n    }"),
    "bulk_columns_pad_zero": ("        bulk_idx[p] = -1;\n", "        bulk_idx[p] = 0;\n"),
    "gather_bulk_by_position": ("w_b[i * k_bulk + p] = bulk_idx[p] < 0 ? 0 : w[i * k + bulk_idx[p]];",
                                "w_b[i * k_bulk + p] = bulk_idx[p] < 0 ? 0 : w[i * k + p];"),
    "gemm_compact_x_by_position": ("double xb = spectra_ref_bf16_to_double(xr[bulk_idx[p]]);",
                                   "double xb = spectra_ref_bf16_to_double(xr[p]);"),
    "gemm_compact_group_of_bulk": ("double wb = ((double)codes[i * k_bulk + p] - (double)zeros[i * Gb + p / 32]) * S;",
                                   "double wb = ((double)codes[i * k_bulk + p] - (double)zeros[i * Gb + p % Gb]) * S;"),
    "pack_outliers_slot_reversed": ("= w[i * k + idx[slot]];", "= w[i * k + idx[n_o - 1 - slot]];"),
    "kv_pack_nibble_swapped": ("(uint8_t)((nib % 2) ? (c << 4) : c);", "(uint8_t)((nib % 2) ? c : (c << 4));"),
    "kv_slot_transposed": ("const int64_t slot = h * cap + pos + t;", "const int64_t slot = t * H + h + pos;"),
    "attention_head_mapping": ("const int64_t h = i / grp;", "const int64_t h = i % Hkv;"),
    "attention_unnormalised": ("o = o + (sc[t] / l) * vv;", "o = o + sc[t] * vv;"),
    "attention_key_zero_index": ("double kv = ((double)kc[slot * D + d] - (double)kz[slot * G + d / 32]) * S;",
                                 "double kv = ((double)kc[slot * D + d] - (double)kz[slot * G + d % G]) * S;"),
    "attention_scale_dropped": ("sc[t] = scale * acc;", "sc[t] = acc;"),
    "row_table_codes_transposed": ("rcodes[(i * G + g) * 16 + word * 4 + j / 2]",
                                   "rcodes[(g * n + i) * 16 + word * 4 + j / 2]"),
    "row_table_scales_transposed": ("rscales[i * G + g] = scales[i * G + g];",
                                    "rscales[g * n + i] = scales[i * G + g];"),
    "row_table_outlier_slot_reversed": ("routl[i * n_o + o] = w[i * kw + idx[o]];",
                                        "routl[i * n_o + o] = w[i * kw + idx[n_o - 1 - o]];"),
    "row_table_outlier_row_stride": ("routl[i * n_o + o] = w[i * kw + idx[o]];",
                                     "routl[i * n_o + o] = w[i * k + idx[o]];"),
    "embed_zero_point_sign": ("dst[col] = ((double)codes[row * k + col] - (double)zeros[grp]) * S;",
                              "dst[col] = ((double)codes[row * k + col] + (double)zeros[grp]) * S;"),
}

PIN_FUNCS = [
    pins.test_fp16_golden_cases,
    pins.test_fp16_random_doubles_match_numpy,
    pins.test_kurtosis_closed_forms,
    pins.test_kurtosis_matches_scipy_with_gain,
    pins.test_split_strict_and_ascending,
    pins.test_quantizer_exact_grid,
    pins.test_quantizer_half_even_ties,
    pins.test_quantizer_invariants_random,
    pins.test_layout_golden_offsets,
    pins.test_layout_roundtrip,
    pins.test_gemm_brute_force_8x32,
    pins.test_gemm_all_outliers_is_dense_product,
    pins.test_gemm_unit_vectors_extract_columns,
    pins.test_bf16_golden_cases,
    pins.test_embed_all_outliers_is_row_indexing,
    pins.test_embed_exact_grid_rows,
    pins.test_embed_rows_agree_with_gemm,
    pins.test_bulk_columns_are_the_complement,
    pins.test_gemm_compact_brute_force_8x64,
    pins.test_gemm_compact_exact_grid_bulk_is_dense_product,
    pins.test_gemm_compact_unit_vectors_extract_columns,
    pins.test_compact_outlier_block_is_the_masked_one,
    pins.test_kv_quantize_is_the_weight_quantiser_per_token,
    pins.test_attention_exact_grid_is_textbook,
    pins.test_attention_one_token_and_zero_query,
    pins.test_kv_pack_golden_offsets,
    pins.test_row_table_golden_offsets,
    pins.test_row_table_rows_are_the_packed_rows,
]
_PARAMS = {
    "test_quantizer_exact_grid": [{"S": 2.0 ** -7, "z": 5}],
    "test_layout_roundtrip": [{"n": 40, "k": 96, "n_o": 9}],
}


def _load_variant(tmp_path, name, old, new):
    d = tmp_path / f"oracle_{name}"
    shutil.copytree(os.path.join(ROOT, "oracle"), d,
                    ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src = d / "spectra_ref.c"
    text = src.read_text()
    assert text.count(old) == 1, f"mutation anchor not unique: {name}"
    src.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_{name}", d / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _caught(mod, golden_dir) -> bool:
    for f in PIN_FUNCS:
        kwargs_list = _PARAMS.get(f.__name__, [{}])
        for kw in kwargs_list:
            args = {"ref": mod}
            if "golden_dir" in f.__code__.co_varnames[:f.__code__.co_argcount]:
                args["golden_dir"] = golden_dir
            try:
                f(**args, **kw)
            except Exception:
                return True
    return False


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, golden_dir, name):
    old, new = MUTATIONS[name]
    mod = _load_variant(tmp_path, name, old, new)
    assert _caught(mod, golden_dir), f"no pin fails for mutation {name}"
