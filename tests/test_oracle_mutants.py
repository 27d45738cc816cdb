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
    for fn in ("oracle_decode", "oracle_append", "oracle_merge", "oracle_num_threads"):
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
