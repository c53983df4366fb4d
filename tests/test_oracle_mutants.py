"""The oracle pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, swaps it in for the real oracle and
checks that at least one pin of tests/test_oracle.py fails.  The real oracle
is restored afterwards.
"""
import os
import subprocess

import pytest

import oracle
import test_oracle as T

SRC = os.path.join(os.path.dirname(oracle.__file__), "pa_oracle.c")

PINS = [
    lambda: T.test_decode_hand_examples(0),
    lambda: T.test_decode_hand_examples(1),
    lambda: T.test_decode_hand_examples(2),
    T.test_decode_seq_len_one_returns_v0_exactly,
    T.test_decode_gqa_maps_consecutive_query_heads_to_one_kv_head,
    lambda: T.test_decode_equal_scores_give_mean_of_v(False),
    lambda: T.test_decode_equal_scores_give_mean_of_v(True),
    T.test_decode_invariant_under_block_permutation,
    T.test_decode_ignores_everything_past_the_sequence_end,
    lambda: T.test_decode_matches_torch_sdpa_on_contiguous_gather(False),
    lambda: T.test_decode_matches_torch_sdpa_on_contiguous_gather(True),
    lambda: T.test_split_merge_equals_single_pass(48),
    T.test_prefill_matches_causal_sdpa,
    T.test_prefill_last_query_equals_decode_of_full_length,
    T.test_e4m3_encode_roundtrip_every_code,
    T.test_e4m3_encode_ties_to_even_and_matches_torch_in_range,
    T.test_e4m3_encode_saturates_and_keeps_nan,
    T.test_e4m3_decode_all_codes_match_torch,
    T.test_write_kv_bf16_places_bits_at_slots_and_touches_nothing_else,
    T.test_write_kv_fp8_codes_match_torch_conversion,
    T.test_copy_blocks_copies_whole_blocks_in_order,
]

# (name, text to find, replacement, how many occurrences to replace)
MUTANTS = [
    ("scale dropped", "s[t] = scale * acc;", "s[t] = acc;", 2),
    ("normaliser dropped", "out[d] /= z;", "out[d] /= 1.0;", 1),
    ("softmax sign flipped", "s[t] = exp(s[t] - m);", "s[t] = exp(m - s[t]);", 1),
    ("gqa mapping modulo", "int kvh = (int)((long)h * Hkv / Hq);", "int kvh = h % Hkv;", 3),
    ("slot uses block index", "t % ORACLE_BLOCK, d, Hkv, D), ks", "(t / ORACLE_BLOCK) % ORACLE_BLOCK, d, Hkv, D), ks", 2),
    ("v read from k cache", "out[d] += s[t] * load_elem(v_cache", "out[d] += s[t] * load_elem(k_cache", 1),
    ("causal bound off by one", "int n = prefix_lens[c] + i + 1;", "int n = prefix_lens[c] + i;", 1),
    ("merge weight ignores max", "double w = lp[p] * exp(mp[p] - M);", "double w = lp[p];", 1),
    ("fp8 scale not applied", "((const uint8_t *)cache)[idx]) * scale;", "((const uint8_t *)cache)[idx]);", 1),
    ("e4m3 truncates", "double n = nearbyint(q);", "double n = floor(q);", 1),
    ("e4m3 exponent bias", "(((e + 7) << 3)", "(((e + 8) << 3)", 1),
    ("fp8 write uses scale, not reciprocal", "float kx = kf * kinv;", "float kx = kf * k_scale[h];", 1),
    ("copy ignores dst", "(char *)k_cache + (size_t)d * block_bytes,", "(char *)k_cache + (size_t)s * block_bytes,", 1),
    ("transposed k index", "cache_index(blk, kvh, t % ORACLE_BLOCK, d, Hkv, D), ks);\n        s[t]",
     "cache_index(blk, kvh, d % ORACLE_BLOCK, t % D, Hkv, D), ks);\n        s[t]", 1),
]


@pytest.fixture(scope="module")
def real_lib():
    return oracle.lib()


@pytest.mark.parametrize("name,find,repl,count", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_pins_catch_planted_mistake(name, find, repl, count, tmp_path, monkeypatch, real_lib):
    src = open(SRC).read()
    assert src.count(find) == count, f"mutation site for '{name}' not found as expected"
    mutated = src.replace(find, repl)
    cpath = tmp_path / "mutant.c"
    cpath.write_text(mutated)
    so = tmp_path / "libmutant.so"
    subprocess.run(["gcc", "-O1", "-std=c11", "-fopenmp", "-fPIC", "-shared", "-o", str(so), str(cpath), "-lm"],
                   check=True)
    monkeypatch.setattr(oracle, "_lib", oracle.load(str(so)))
    failed = []
    for pin in PINS:
        try:
            pin()
        except Exception as e:  # noqa: BLE001 -- any failure of a pin counts
            failed.append(type(e).__name__)
    assert failed, f"no pin caught the planted mistake '{name}'"
