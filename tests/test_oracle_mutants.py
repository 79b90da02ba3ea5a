"""The oracle's pins must catch plausible mistakes. Each case plants one mistake in a private copy of
the oracle source (on the CPU, in a temporary directory), builds it, and checks that at least one pin
from ``test_oracle_pins`` fails on the planted copy. The real oracle is never modified.
"""
import importlib.util
import os
import shutil
import sys

import pytest

import test_oracle_pins as pins

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

# (name, text to replace, replacement, pins expected to notice)
MUTANTS = [
    ("dropped_key_zero_point",
     "    out[ch] = static_cast<double>(code) * s + z;\n  }\n  if (c->outliers) {  // the token's fp16 outlier replaces its entry (reading R12)\n    const uint16_t ch = cache->k_out_ch",
     "    out[ch] = static_cast<double>(code) * s + 0.0 * z;\n  }\n  if (c->outliers) {  // the token's fp16 outlier replaces its entry (reading R12)\n    const uint16_t ch = cache->k_out_ch",
     ["test_quantized_attention_equals_library_attention_on_dequantized_cache"]),
    ("hadamard_sign_flip",
     "        x[i] = a + b;\n        x[i + h] = a - b;\n      }\n  const float s",
     "        x[i] = a + b;\n        x[i + h] = b - a;\n      }\n  const float s",
     ["test_wht_f32_scale_constant_and_accuracy", "test_hadamard_no_quantization_equals_rotated_attention"]),
    ("truncating_instead_of_rounding",
     "float r = std::nearbyint(v);", "float r = std::floor(v);",
     ["test_quantizer_invariants", "test_quantizer_half_way_ties_go_to_even"]),
    ("wrong_level_count",
     "const float levels = static_cast<float>((1 << bits) - 1);",
     "const float levels = static_cast<float>(1 << bits);",
     ["test_quantizer_invariants", "test_quantizer_two_valued_and_grid_round_trip"]),
    ("transposed_key_fragment",
     "  const int lane = 4 * r + qd;\n  const int p = 4 * m + (u + 2 * h);\n  slot_to_word_bit(lane, p, bits, e, word, bit);\n}\n\nvoid value_word_bit",
     "  const int lane = 4 * r + qd;\n  const int p = 4 * m + (2 * u + h);\n  slot_to_word_bit(lane, p, bits, e, word, bit);\n}\n\nvoid value_word_bit",
     ["test_layout_matches_hand_worked_examples"]),
    ("softmax_not_normalized",
     "    l += p;\n", "    l += 0.5 * p;\n",
     ["test_no_quantization_equals_library_attention", "test_single_token_returns_its_value"]),
    ("wrong_gqa_head_map",
     "  const int64_t kvh = h / gq;", "  const int64_t kvh = h % c->num_kv_heads;",
     ["test_no_quantization_equals_library_attention"]),
    ("signed_zero_order_reversed",
     "return (h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u);",
     "return (h == 0x8000u) ? 0x8001u : ((h & 0x8000u) ? (~h & 0xffffu) : (h | 0x8000u));",
     ["test_quantizer_signed_zero_minimum"]),
    ("residual_window_rounded_up",
     "return over > 0 ? (over / G) * G : 0;", "return over > 0 ? ((over + G - 1) / G) * G : 0;",
     ["test_quantized_attention_equals_library_attention_on_dequantized_cache"]),
    ("rows_v2_value_words_swapped",
     "  *word = (block * 128 + c) * (4 * bits) + j / P;",
     "  *word = (block * 128 + c) * (4 * bits) + ((j / P) ^ 1);",
     ["test_layout_matches_hand_worked_examples"]),
    ("sink_first_token_in_group_zero_stats",
     "  const int skip = (c->sink && t0 == 0) ? 1 : 0;", "  const int skip = 0;",
     ["test_sink_first_token_left_out_of_group_zero"]),
    ("sink_row_ignored_by_decode",
     "  if (t >= Q || (c->sink && t == 0)) {\n    const int64_t row = (c->sink && t == 0) ? d.ring : t % d.ring;\n    const uint16_t* r = cache->k_res",
     "  if (t >= Q) {\n    const int64_t row = (c->sink && t == 0) ? d.ring : t % d.ring;\n    const uint16_t* r = cache->k_res",
     ["test_sink_dominant_first_token_returns_its_fp16_value"]),
    ("rope_sin_sign_flipped",
     "    k[i] = a * cs - b * sn;", "    k[i] = a * cs + b * sn;",
     ["test_rope_without_quantization_equals_library_attention_on_rotated_keys"]),
    ("rope_frequency_exponent_halved",
     "std::pow(static_cast<double>(c->rope_theta), -i / 64.0)",
     "std::pow(static_cast<double>(c->rope_theta), -i / 128.0)",
     ["test_rope_without_quantization_equals_library_attention_on_rotated_keys"]),
    ("rope_position_off_by_one",
     "    if (rope) rope_rotate(row, t, omega);", "    if (rope) rope_rotate(row, t + 1, omega);",
     ["test_rope_without_quantization_equals_library_attention_on_rotated_keys", "test_rope_relative_position"]),
    ("outliers_kept_in_key_statistics",
     "kc.data() + skip * 128 + ch, 128, kout.data() + skip * 128 + ch, 128);",
     "kc.data() + skip * 128 + ch, 128);",
     ["test_outliers_left_out_of_group_statistics"]),
    ("value_outlier_not_restored_in_decode",
     "    if (ch < 128) out[ch] = half_to_float(cache->v_out_val[slot * d.slot_tokens + ts]);",
     "    (void)ch;",
     ["test_outliers_dequantized_attention_equals_library_attention"]),
    ("page_table_row_stride_dropped",
     "  *slot = cache->page_table[unit * pages_per_unit + t / c->page_tokens];",
     "  *slot = cache->page_table[unit + t / c->page_tokens];",
     ["test_paged_shuffled_pool_gathers_to_the_contiguous_cache"]),
    ("value_read_skips_the_page_table",
     "  int64_t slot, ts;  // where token t is stored (reading R13)\n  locate(c, cache, unit, t, &slot, &ts);\n  const uint32_t* vbuf",
     "  int64_t slot = unit, ts = t;\n  const uint32_t* vbuf",
     ["test_paged_shuffled_pool_gathers_to_the_contiguous_cache"]),
    ("outlier_ties_to_the_highest_channel",
     "    if ((x[ch] & 0x7fffu) > (x[best] & 0x7fffu)) best = ch;",
     "    if ((x[ch] & 0x7fffu) >= (x[best] & 0x7fffu)) best = ch;",
     ["test_outliers_are_each_tokens_largest_entry_kept_in_fp16"]),
    ("value_group_index_off",
     "    const int j = ch / c->group_size;", "    const int j = (ch / c->group_size + 1) % d.vpt;",
     ["test_quantized_attention_equals_library_attention_on_dequantized_cache"]),
]


def _load_mutant(tmp_path, name, old, new):
    dst = tmp_path / f"oracle_{name}"
    shutil.copytree(os.path.join(ROOT, "oracle"), dst, ignore=shutil.ignore_patterns("*.so", "__pycache__"))
    src = dst / "kvq_oracle.cpp"
    text = src.read_text()
    assert text.count(old) == 1, f"mutation anchor for {name} not found exactly once"
    src.write_text(text.replace(old, new))
    spec = importlib.util.spec_from_file_location(f"oracle_mutant_{name}", dst / "__init__.py")
    mod = importlib.util.module_from_spec(spec)
    sys.modules[spec.name] = mod
    spec.loader.exec_module(mod)
    mod.build(force=True)
    return mod


def _run_pin(fn_name, mod):
    fn = getattr(pins, fn_name)
    params = {
        "test_quantizer_invariants": [dict(bits=2, G=32), dict(bits=4, G=16)],
        "test_quantizer_two_valued_and_grid_round_trip": [dict(bits=2), dict(bits=4)],
        "test_quantized_attention_equals_library_attention_on_dequantized_cache":
            [dict(kb=2, vb=2, G=32, R=32, had=0, layout=1), dict(kb=2, vb=2, G=32, R=32, had=0, layout=2)],
        "test_sink_first_token_left_out_of_group_zero": [dict(layout=1), dict(layout=2)],
        "test_sink_dominant_first_token_returns_its_fp16_value": [dict(layout=1), dict(layout=2)],
        "test_rope_without_quantization_equals_library_attention_on_rotated_keys": [dict(theta=10000.0)],
        "test_outliers_left_out_of_group_statistics": [dict(layout=1)],
        "test_outliers_are_each_tokens_largest_entry_kept_in_fp16": [dict(layout=1)],
        # all of the pool's table entries are valid pages here, so a wrong lookup stays in bounds
        "test_paged_shuffled_pool_gathers_to_the_contiguous_cache": [dict(layout=1, outliers=0)],
    }.get(fn_name, [dict()])
    for kw in params:
        fn(mod, **kw)


@pytest.mark.parametrize("name,old,new,catchers", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(tmp_path, name, old, new, catchers):
    mod = _load_mutant(tmp_path, name, old, new)
    caught = []
    for fn_name in catchers:
        try:
            _run_pin(fn_name, mod)
        except AssertionError:
            caught.append(fn_name)
    assert caught, f"no pin noticed the planted mistake {name}"
