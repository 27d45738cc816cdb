"""Plant plausible slips in a COPY of the oracle (on the CPU) and check that
the pins in test_oracle_pins.py catch every one of them.

Each mutant is a one-token change to oracle.c that keeps every memory access
in bounds; it is compiled into a temporary library that stands in for the
real one while the pins run.
"""
import ctypes
import os
import subprocess

import pytest

import oracle
import test_oracle_append_attn as aapins
import test_oracle_fp8 as fp8pins
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "oracle.c")

MUTANTS = {
    "head_mapping": ("const int g = h / group;", "const int g = h % num_kv_heads;"),
    "keys_read_from_values": ("pool_offset(page, 0, g, t % page_size,",
                              "pool_offset(page, 1, g, t % page_size,"),
    "no_max_subtraction": ("const double w = exp(s[t] - m);", "const double w = exp(s[t]);"),
    "lse_drops_max": ("lse[row] = m + log(l);", "lse[row] = log(l);"),
    "ignores_last_page_len": ("return (np - 1) * (int64_t)page_size + last_page_len[b];",
                              "return np * (int64_t)page_size;"),
    "scale_dropped": ("s[t] = scale * dot;", "s[t] = dot;"),
    "f16_exponent_bias": ("e - 25);", "e - 24);"),
    "merge_lse_unshifted": ("const double w = exp(sj - m);", "const double w = exp(sj - 0.5 * m);"),
    "append_slot_shift": ("const int64_t slot = pos % page_size;",
                          "const int64_t slot = (pos + 1) % page_size;"),
    "append_page_of_next": ("page_indices[page_indptr[b] + pos / page_size];\n      const int64_t slot",
                            "page_indices[page_indptr[b] + (pos / page_size + 1) % (page_indptr[b + 1] - page_indptr[b])];\n      const int64_t slot"),
    "e4m3_exponent_bias": ("ldexp((double)(frac | 8), e - 10)", "ldexp((double)(frac | 8), e - 9)"),
    "e4m3_subnormal_scale": ("if (e == 0) v = ldexp((double)frac, -9);",
                             "if (e == 0) v = ldexp((double)frac, -10);"),
    "e4m3_ties_to_odd": ("(c & 1) == 0", "(c & 1) == 1"),
    "e4m3_saturates_to_nan": ("(uint8_t)((neg << 7) | 0x7e)", "(uint8_t)((neg << 7) | 0x7f)"),
    "e4m3_scale_multiplies": ("const float q = x / scale;", "const float q = x * scale;"),
    "fp8_keys_take_v_scale": ("(kv_elem(pool, kv_dtype, k + d) * k_scale)",
                              "(kv_elem(pool, kv_dtype, k + d) * v_scale)"),
    "fp8_values_unscaled": ("(kv_elem(pool, kv_dtype, v + d) * v_scale)",
                            "(kv_elem(pool, kv_dtype, v + d))"),
    "fp8_append_v_takes_k_scale": ("encode_e4m3((float)widen(vs[d], new_dtype), v_scale)",
                                   "encode_e4m3((float)widen(vs[d], new_dtype), k_scale)"),
    "e5m2_exponent_bias": ("ldexp((double)(frac | 4), e - 17)", "ldexp((double)(frac | 4), e - 16)"),
    "e5m2_ties_to_odd": ("(err == best_err && !(c & 1))", "(err == best_err && (c & 1))"),
    "e5m2_saturates_to_inf": ("(uint8_t)((neg << 7) | 0x7b)", "(uint8_t)((neg << 7) | 0x7c)"),
    "chunk_not_causal_on_self": ("if (t > pos) return 0;", "if (t >= pos && pos > 0) return 0;"),
    "chunk_window_one_short": ("return t >= pos - window_left ||", "return t > pos - window_left ||"),
    "chunk_head_mapping": ("const int kvh = h / group;", "const int kvh = h % num_kv_heads;"),
    "chunk_sink_ignored": ("return t >= pos - window_left || t < sink_tokens;",
                           "return t >= pos - window_left;"),
    "chunk_positions_from_zero": ("const int64_t pos = len - n_q + (r - qo_indptr[b]);",
                                  "const int64_t pos = len - n_q + (r - qo_indptr[b]) - 1 + (n_q == 1);"),
}

PINS = [
    lambda: [pins.test_oracle_matches_dense_sdpa(c) for c in range(len(pins.CASES))],
    pins.test_large_logits_need_max_subtraction,
    lambda: pins.test_single_token_returns_its_value_exactly("f16"),
    lambda: pins.test_single_token_returns_its_value_exactly("bf16"),
    pins.test_identical_keys_give_mean_of_values,
    pins.test_zero_query_gives_mean_of_values_and_value_shift,
    pins.test_hand_derived_tiny_cases,
    pins.test_empty_request_and_canaries,
    pins.test_merge_of_split_sequence_equals_whole,
    pins.test_merge_closed_forms,
    pins.test_append_hand_derived_positions,
    pins.test_append_extends_the_logical_sequence,
    fp8pins.test_code_values_from_the_format_definition,
    fp8pins.test_encode_matches_torch_round_to_nearest_even,
    fp8pins.test_encode_saturates_and_keeps_nan,
    fp8pins.test_encode_divides_by_the_scale_in_binary32,
    lambda: [fp8pins.test_fp8_decode_matches_dense_sdpa_on_dequantised_values(c)
             for c in range(len(fp8pins.FP8_CASES))],
    lambda: fp8pins.test_fp8_append_positions_and_codes("e4m3"),
    lambda: fp8pins.test_fp8_append_positions_and_codes("e5m2"),
    fp8pins.test_e5m2_code_values_from_the_format_definition,
    fp8pins.test_e5m2_encode_matches_torch_and_saturates,
    lambda: [aapins.test_append_attention_matches_masked_sdpa(c) for c in range(len(aapins.CASES))],
    aapins.test_single_token_chunks_are_the_decode,
    aapins.test_chunking_invariance,
    aapins.test_hand_derived_identical_keys_and_windows,
]


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path, monkeypatch):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) == 1, f"mutation anchor for {name} not unique"
    src = tmp_path / "mutant.c"
    src.write_text(text.replace(old, new))
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(src),
                    "-o", str(so), "-lm"], check=True)
    real = oracle._load()
    lib = ctypes.CDLL(str(so))
    for fn in ("oracle_decode", "oracle_append", "oracle_merge", "oracle_num_threads",
               "oracle_decode_fp8", "oracle_append_fp8", "oracle_e4m3_decode",
               "oracle_e4m3_encode", "oracle_append_attention", "oracle_e5m2_decode",
               "oracle_e5m2_encode"):
        getattr(lib, fn).argtypes = getattr(real, fn).argtypes
        getattr(lib, fn).restype = getattr(real, fn).restype
    monkeypatch.setattr(oracle, "_lib", lib)
    caught = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, oracle.OracleError):
            caught.append(pin)
    assert caught, f"no pin caught mutant {name}"
