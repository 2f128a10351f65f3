"""Plant plausible mistakes in a copy of the oracle's C source and check that
the pins in test_oracle_pins.py catch every one of them (CPU only)."""
import os

import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")

# (name, exact text in pkv_oracle.c, replacement)
MUTANTS = [
    ("drop_scale", "s[i] = scale * dot;", "s[i] = dot;"),
    ("no_max_shift", "s[i] = exp(s[i] - m);", "s[i] = exp(s[i]);"),
    ("gqa_modulo", "h / G", "h % num_kv_heads"),
    ("page_index_mod", "+ i / c->page_size];", "+ i % c->page_size];"),
    ("slot_offset_div", "+ i % c->page_size;", "+ i / c->page_size;"),
    ("causal_off_by_one", "causal ? pos + 1 : ctx", "causal ? pos : ctx"),
    ("top_left_alignment", "int pos = ctx - n + r;", "int pos = r;"),
    ("no_normalise", "out[d] = acc / L;", "out[d] = acc;"),
    ("pool_head_major", "int64_t row = slot * c->num_kv_heads + kvh;",
     "int64_t row = (int64_t)kvh * c->num_pages * c->page_size + slot;"),
    ("values_from_k_pool", "acc += s[i] * or_kv(c, 1,", "acc += s[i] * or_kv(c, 0,"),
    ("v_uses_k_scales", "(is_v ? c->v_scales : c->k_scales)", "(c->k_scales)"),
    ("quant_truncates", "rintf(v / s)", "truncf(v / s)"),
    ("quant_divides_by_128", "a / 127.0f", "a / 128.0f"),
    ("quant_no_clamp", "if (t > 127.0f) t = 127.0f;", ""),
    ("lse_sign", "*lse = m + log(L);", "*lse = m - log(L);"),
    ("f16_exponent_bias", "e - 25", "e - 24"),
    ("f16_round_truncates", "double r = rint(ldexp(a, 10 - E));", "double r = floor(ldexp(a, 10 - E));"),
    ("bf16_shift", "(uint32_t)b << 16", "(uint32_t)b << 15"),
    ("scatter_swaps_kv", "(const char*)v + t * row_bytes", "(const char*)k + t * row_bytes"),
    ("window_off_by_one", "pos - window + 1 > 0) ? pos - window + 1 : 0", "pos - window > 0) ? pos - window : 0"),
    ("decode_window_ignored", "(window > 0 && ctx - window > 0) ? ctx - window : 0", "0"),
    ("window_only_when_causal", "int k_lo = (window > 0 && pos", "int k_lo = (window > 0 && causal && pos"),
    ("window_band_from_context_end", "pos - window + 1 > 0) ? pos - window + 1 : 0",
     "k_hi - window > 0) ? k_hi - window : 0"),
]

CHECKS = [
    pins.test_golden_decode_closed_form,
    pins.test_golden_int8_quant_rows,
    pins.test_single_token_context_returns_v_exactly,
    pins.test_constant_v_gives_constant_output,
    pins.test_page_permutation_invariance_is_bitwise,
    lambda: pins.test_paged_equals_contiguous_sdpa("f64"),
    lambda: pins.test_paged_equals_contiguous_sdpa("bf16"),
    pins.test_shared_prefix_equals_private_copies_bitwise,
    pins.test_brute_force_tiny,
    pins.test_one_hot_query_large_scale_picks_argmax_value,
    pins.test_zero_query_gives_mean_of_values,
    pins.test_gqa_contiguous_group_mapping,
    pins.test_lse_matches_torch_logsumexp,
    pins.test_split_kv_merge_algebra,
    pins.test_int8_dequant_path_equals_explicit_dequant,
    lambda: pins.test_prefill_matches_sdpa_bottom_right(True),
    lambda: pins.test_prefill_matches_sdpa_bottom_right(False),
    pins.test_prefill_last_row_equals_decode_and_first_row_without_prefix,
    pins.test_quantiser_bounds_and_symmetry,
    pins.test_scatter_matches_fancy_index_assignment,
    pins.test_f16_widening_and_rounding_match_numpy,
    pins.test_bf16_widening_matches_torch_for_all_patterns,
    pins.test_window_covering_the_context_equals_no_window,
    pins.test_window_one_returns_the_own_value,
    lambda: pins.test_window_matches_sdpa_band_mask(3, True),
    lambda: pins.test_window_matches_sdpa_band_mask(3, False),
]


@pytest.mark.parametrize("name,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_mutant(tmp_path, name, old, new):
    text = open(SRC).read()
    assert old in text, f"mutation site for {name} not found"
    src = tmp_path / f"{name}.c"
    src.write_text(text.replace(old, new))
    lib = oracle.build(force=True, src=str(src), out=str(tmp_path / f"{name}.so"))
    caught = None
    with oracle.using_library(lib):
        for check in CHECKS:
            try:
                check()
            except (AssertionError, ValueError) as e:
                caught = e
                break
    assert caught is not None, f"no pin caught mutant {name}"
