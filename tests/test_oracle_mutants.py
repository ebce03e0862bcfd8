"""Plant one plausible mistake at a time in a copy of the oracle's C source and
check that the pins in test_oracle_pins.py reject every such copy.  Runs on the
CPU only; the real oracle is never modified."""
import os

import pytest

import oracle
from tests import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "dsa_oracle.c")

# (name, original text, mutated text); each original must occur exactly once
MUTANTS = [
    ("relu dropped", "double relu = dot > 0.0 ? dot : 0.0;", "double relu = dot;"),
    ("causal mask excludes the diagonal", "      if (s > pos) {\n        out[s] = -INFINITY;",
     "      if (s >= pos) {\n        out[s] = -INFINITY;"),
    ("sequence offset of key rows dropped", "int64_t key_row = cu_k[b] + s;", "int64_t key_row = s;"),
    ("head weight of the wrong query", "total += w[t * H_I + j] * relu;", "total += w[j] * relu;"),
    ("e4m3 exponent bias off by one", "v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);"),
    ("e4m3 subnormal scale", "v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    ("e4m3 scale not applied", "* (double)row_scale[row];", ";"),
    ("bf16 bits misplaced", "uint32_t u = ((uint32_t)bits) << 16;", "uint32_t u = ((uint32_t)bits) << 15;"),
    ("tie-break reversed", "return (x->index > y->index) - (x->index < y->index);",
     "return (x->index < y->index) - (x->index > y->index);"),
    ("ascending instead of descending", "if (x->score > y->score) return -1;\n  if (x->score < y->score) return 1;",
     "if (x->score > y->score) return 1;\n  if (x->score < y->score) return -1;"),
    ("diagonal candidate dropped", "int64_t n = pos + 1;\n    candidate*", "int64_t n = pos;\n    candidate*"),
    ("softmax scale dropped", "z[i] = scale * dot;", "z[i] = dot;"),
    ("values from the tail of the latent row",
     "for (int d = 0; d < d_v; ++d) o[d] += p * load_elem(c_kind, latent, row * d_qk + d, NULL, 0);\n      }\n      lse[r * H + h] = zmax + log(denom);\n    }\n    free(z);",
     "for (int d = 0; d < d_v; ++d) o[d] += p * load_elem(c_kind, latent, row * d_qk + (d_qk - d_v) + d, NULL, 0);\n      }\n      lse[r * H + h] = zmax + log(denom);\n    }\n    free(z);"),
    ("lse without the max", "      lse[r * H + h] = zmax + log(denom);\n    }\n    free(z);",
     "      lse[r * H + h] = log(denom);\n    }\n    free(z);"),
    ("causal check of selected entries off by one", "return s >= 0 && s <= pos && s < kv_len;",
     "return s >= 0 && s <= pos + 1 && s < kv_len;"),
    ("query head stride wrong", "dot += load_elem(q_kind, q, (t * H + h) * (int64_t)d_qk + d, NULL, 0) *\n                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);\n        z[i]",
     "dot += load_elem(q_kind, q, (t * H) * (int64_t)d_qk + d, NULL, 0) *\n                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);\n        z[i]"),
    # FP8 indexer: rotation, encoding, scales
    ("Hadamard signs dropped", "acc += sign ? -x[v * d + j] : x[v * d + j];", "acc += x[v * d + j];"),
    ("Hadamard not normalised", "y[v * d + i] = acc * norm;", "y[v * d + i] = acc;"),
    ("e4m3 ties to odd", "(err == best_err && (code & 1) == 0)", "(err == best_err && (code & 1) == 1)"),
    ("e4m3 sign dropped", "return (uint8_t)(best | (neg << 7));", "return (uint8_t)best;"),
    ("power-of-two scale rounded down", "ldexp(1.0, (int)ceil(log2(amax / 448.0)))",
     "ldexp(1.0, (int)floor(log2(amax / 448.0)))"),
    ("query scale of the wrong head", "(t * H_I + j) * (int64_t)d_I + d, q_scale, t * H_I + j);",
     "(t * H_I + j) * (int64_t)d_I + d, q_scale, t * H_I);"),
    # rotary embedding
    ("rotation sign", "y[v * d + 2 * i] = re * c - im * s;", "y[v * d + 2 * i] = re * c + im * s;"),
    ("pair halves swapped", "const double re = x[v * d + 2 * i], im = x[v * d + 2 * i + 1];",
     "const double re = x[v * d + 2 * i + 1], im = x[v * d + 2 * i];"),
    # paged layout and append quantization
    ("row inside the page taken from the wrong end", "r = (page >= 0 && page < n_pages) ? page * page_size + s % page_size : -1;",
     "r = (page >= 0 && page < n_pages) ? page * page_size + (page_size - 1 - s % page_size) : -1;"),
    ("page table row stride dropped", "block_table[(int64_t)b * pages_per_seq + j]", "block_table[j]"),
    ("pages beyond the pool accepted", "r = (page >= 0 && page < n_pages) ?", "r = (page >= 0) ?"),
    ("amax scale of the wrong format maximum", "(float)(amax / 448.0)", "(float)(amax / 240.0)"),
    # up-projection
    ("up-projection matrix transposed", "load_elem(w_kind, w, ((int64_t)h * d_c + c) * d_v + e, NULL, 0);",
     "load_elem(w_kind, w, ((int64_t)h * d_v + e) * d_c + c, NULL, 0);"),
    ("up-projection reads head 0 of the output", "acc += o[(r * H + h) * (int64_t)d_c + c]",
     "acc += o[(r * H) * (int64_t)d_c + c]"),
    # more slips of the three steps (every mutated index stays inside its array)
    ("query position counted from the start of the cache", "*pos_out = kv_len - q_len + (t - cu_q[b]);",
     "*pos_out = t - cu_q[b];"),
    ("key scale taken by the sequence-local index", "load_elem(k_kind, k_idx, key_row * d_I + d, k_scale, key_row);",
     "load_elem(k_kind, k_idx, key_row * d_I + d, k_scale, s);"),
    ("top-k padded with index 0", "idx[r * topk + i] = i < keep ? c[i].index : -1;",
     "idx[r * topk + i] = i < keep ? c[i].index : 0;"),
    ("QK reduced over the value columns only",
     "for (int d = 0; d < d_qk; ++d)\n          dot += load_elem(q_kind, q, (t * H + h) * (int64_t)d_qk + d, NULL, 0) *\n"
     "                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);\n        z[i]",
     "for (int d = 0; d < d_v; ++d)\n          dot += load_elem(q_kind, q, (t * H + h) * (int64_t)d_qk + d, NULL, 0) *\n"
     "                 load_elem(c_kind, latent, row * d_qk + d, NULL, 0);\n        z[i]"),
    ("softmax numerator without the max", "double p = exp(z[i] - zmax) / denom;", "double p = exp(z[i]) / denom;"),
    ("e4m3 mantissa read as four bits", "v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 16.0, e - 7);"),
    ("Hadamard normalised by 1/d", "1.0 / sqrt((double)d)", "1.0 / (double)d"),
    ("RoPE table pairs in reverse order",
     "const double c = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 0];\n"
     "      const double s = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 1];",
     "const double c = freqs[((int64_t)pos[v] * (d / 2) + (d / 2 - 1 - i)) * 2 + 0];\n"
     "      const double s = freqs[((int64_t)pos[v] * (d / 2) + (d / 2 - 1 - i)) * 2 + 1];"),
    ("RoPE cos and sin swapped",
     "const double c = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 0];\n"
     "      const double s = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 1];",
     "const double c = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 1];\n"
     "      const double s = freqs[((int64_t)pos[v] * (d / 2) + i) * 2 + 0];"),
    ("power-of-two scale from the signed maximum",
     "amax = fmax(amax, fabs(x[v * d + i]));\n    const double s",
     "amax = fmax(amax, x[v * d + i]);\n    const double s"),
    ("amax scale from the signed maximum",
     "amax = fmax(amax, fabs(x[v * d + i]));\n    const float s",
     "amax = fmax(amax, x[v * d + i]);\n    const float s"),
]

from tests import test_oracle_pins_cache as pins_cache
from tests import test_oracle_pins_ext as pins_ext

PIN_TESTS = [
    ("test_e4m3_decode_exhaustive", {}),
    ("test_bf16_decode_random_patterns", {}),
    ("test_scores_match_einsum", {"kfp8": False}),
    ("test_scores_match_einsum", {"kfp8": True}),
    ("test_scores_exact_on_integer_inputs", {}),
    ("test_hadamard_rotation_leaves_scores_unchanged", {}),
    ("test_topk_matches_lexsort_with_ties", {"levels": 3}),
    ("test_topk_invariants", {}),
    ("test_sparse_equals_dense_causal_when_topk_covers_everything", {}),
    ("test_sparse_equals_additive_mask_formulation", {}),
    ("test_attention_closed_forms", {}),
    ("test_attention_ignores_order_padding_and_invalid_entries", {}),
]

PIN_TESTS_EXT = [
    ("test_hadamard_is_the_normalised_sylvester_matrix", {"d": 32}),
    ("test_e4m3_encoding_round_trips_every_finite_code", {}),
    ("test_e4m3_encoding_matches_torch_round_to_nearest_even", {}),
    ("test_quantization_scale_is_the_smallest_power_of_two_that_fits", {}),
    ("test_fp8_scores_match_einsum_of_the_dequantized_values", {}),
    ("test_rope_is_complex_multiplication_by_the_table", {}),
    ("test_rope_closed_forms", {}),
    ("test_up_projection_matches_einsum_and_selects_with_a_unit_matrix", {}),
]

PIN_TESTS_CACHE = [
    ("test_paged_rows_worked_example", {}),
    ("test_packed_layout_is_the_identity", {}),
    ("test_paged_rows_agree_with_a_pool_filled_page_by_page", {}),
    ("test_paged_rows_mark_missing_pages", {}),
    ("test_amax_quantization_matches_float32_division_and_torch_cast", {}),
    ("test_append_decode_rows_are_the_last_rows_and_rope_closed_forms", {}),
    ("test_append_prefill_rows_and_paging", {}),
]


def _caught(lib_mod):
    for module, tests in ((pins, PIN_TESTS), (pins_ext, PIN_TESTS_EXT), (pins_cache, PIN_TESTS_CACHE)):
        for name, kw in tests:
            try:
                getattr(module, name)(lib_mod, **kw)
            except Exception:
                return name
    return None


def test_unmutated_copy_passes_every_pin(tmp_path):
    so = oracle.compile_source(SRC, str(tmp_path / "copy.so"))
    with oracle.use_library(so):
        assert _caught(oracle) is None


@pytest.mark.parametrize("name,orig,mut", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_reject_mutant(tmp_path, name, orig, mut):
    src = open(SRC).read()
    assert src.count(orig) == 1, f"mutation site not unique: {name}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(orig, mut))
    so = oracle.compile_source(str(path), str(tmp_path / "mutant.so"))
    with oracle.use_library(so):
        caught_by = _caught(oracle)
    assert caught_by is not None, f"no pin rejects the mutant '{name}'"
