"""Pin strength: copies of the oracle with one planted mistake each must fail a pin.

Each mutation edits a private copy of ``oracle/pa_oracle.c`` under a temporary
directory and builds it there; the committed oracle is never touched. Only
mutations that keep every memory access in bounds are planted.
"""
import os

import pytest

import oracle
from tests import oracle_pins

MUTATIONS = {
    "gqa_mapping": ("const int kvh = h / group;", "const int kvh = h % num_kv_heads;"),
    "f16_exponent": ("mag = ldexp((double)(m + 1024), e - 25);",
                     "mag = ldexp((double)(m + 1024), e - 24);"),
    "bf16_exponent": ("mag = ldexp((double)(m + 128), e - 134);",
                      "mag = ldexp((double)(m + 128), e - 133);"),
    "f16_subnormal": ("mag = ldexp((double)m, -24);", "mag = ldexp((double)m, -25);"),
    "bf16_subnormal": ("mag = ldexp((double)m, -133);", "mag = ldexp((double)m, -132);"),
    "sign_dropped": ("return sign ? -mag : mag;", "return mag;"),
    "scale_dropped": ("scores[t] = exp(scale * scores[t] - mx);", "scores[t] = exp(scores[t] - mx);"),
    "key_index_reversed": ("dot += qd[d] * oracle_to_double(key[d], dtype);",
                           "dot += qd[d] * oracle_to_double(key[head_dim - 1 - d], dtype);"),
    "values_from_key_pool": ("v_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;",
                             "k_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;"),
    "key_row_swapped": ("k_pool + ((page * num_kv_heads + kvh) * block_size + r) * head_dim;",
                        "k_pool + ((page * num_kv_heads + kvh) * block_size + (r ^ 1)) * head_dim;"),
    "no_normalisation": ("scores[t] /= total;", "scores[t] /= 1.0;"),
    "table_ignored": ("const size_t page = (size_t)table[i];", "const size_t page = (size_t)i;"),
    "query_head_0": ("qd[d] = oracle_to_double(q[(size_t)sh * head_dim + d], dtype);",
                     "qd[d] = oracle_to_double(q[(size_t)s * num_heads * head_dim + d], dtype);"),
    "last_token_dropped": ("const int n = context_lens[s];",
                           "const int n = context_lens[s] - (context_lens[s] > 1);"),
    "cache_offset": ("const int64_t offset = slot % block_size;",
                     "const int64_t offset = (slot + 1) % block_size;"),
    "cache_head_swapped": ("const size_t src = ((size_t)t * num_kv_heads + h) * head_dim;",
                           "const size_t src = ((size_t)t * num_kv_heads + (num_kv_heads - 1 - h)) * head_dim;"),
    "copy_direction": ("const int64_t src = src_dst_pairs[2 * p];\n        const int64_t dst = src_dst_pairs[2 * p + 1];",
                       "const int64_t src = src_dst_pairs[2 * p + 1];\n        const int64_t dst = src_dst_pairs[2 * p];"),
    "swap_pool_index": ("memcpy(dst_pools[i] + (size_t)dst * block_bytes,\n                   src_pools[i] + (size_t)src * block_bytes, block_bytes);",
                        "memcpy(dst_pools[i] + (size_t)dst * block_bytes,\n                   src_pools[num_pools - 1 - i] + (size_t)src * block_bytes, block_bytes);"),
    "e4m3_bias": ("mag = ldexp((double)(m + 8), e - 10);", "mag = ldexp((double)(m + 8), e - 11);"),
    "e4m3_subnormal_step": ("mag = ldexp((double)m, -9);", "mag = ldexp((double)m, -10);"),
    "e4m3_ties_away": ("if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) == 1.0))\n        r += 1.0;\n    if (r == 16.0)",
                       "if (f >= 0.5)\n        r += 1.0;\n    if (r == 16.0)"),
    "e4m3_saturation": ("if (a >= 464.0)                         /* rounds past 448: saturate */\n        return sign | 0x7e;",
                        "if (a >= 464.0)                         /* rounds past 448: saturate */\n        return sign | 0x7d;"),
    "fp8_key_scale_dropped": ("dot += qd[d] * (k_scale * oracle_e4m3_to_double(key[d]));",
                              "dot += qd[d] * oracle_e4m3_to_double(key[d]);"),
    "fp8_value_scale_dropped": ("o[d] += scores[t] * (v_scale * oracle_e4m3_to_double(val[d]));",
                                "o[d] += scores[t] * oracle_e4m3_to_double(val[d]);"),
    "fp8_write_scale_times": ("k_pool[dst + d] = oracle_e4m3_encode(kx / k_scale);",
                              "k_pool[dst + d] = oracle_e4m3_encode(kx * k_scale);"),
    "int8_excess_127": ("return (double)code - 128.0;", "return (double)code - 127.0;"),
    "int8_ties_away": ("if (f > 0.5 || (f == 0.5 && fmod(r, 2.0) != 0.0))", "if (f >= 0.5)"),
    "int8_clamps_at_minus_128": ("if (y <= -127.0f)\n        return 1;", "if (y <= -127.0f)\n        return 0;"),
    "kv8_scale_of_query_head": ("const double ks = kv8_scale(k_scales, per_block, page, kvh, num_kv_heads);",
                                "const double ks = kv8_scale(k_scales, per_block, page, h % num_kv_heads, "
                                "num_kv_heads);"),
    "kv8_scales_swapped": ("const double ks = kv8_scale(k_scales, per_block, page, kvh, num_kv_heads);",
                           "const double ks = kv8_scale(v_scales, per_block, page, kvh, num_kv_heads);"),
    "kv8_write_scale_of_head_0": ("/ k_scales[si];", "/ k_scales[0];"),
    "kv8_block_scale_of_head": ("return per_block ? scales[page * (size_t)num_kv_heads + kvh] : scales[kvh];",
                                "return per_block ? scales[kvh] : scales[kvh];"),
    "kv8_write_block_scale_of_head": (
        "const size_t si = per_block ? (size_t)block * num_kv_heads + h : (size_t)h;",
        "const size_t si = (size_t)h;"),
    "kv8_format_ignored": (
        "return format == ORACLE_KV_INT8 ? oracle_int8_to_double(code) : oracle_e4m3_to_double(code);",
        "return oracle_e4m3_to_double(code);"),
    "negative_slot_stops_the_write": (
        "int num_kv_heads, int head_dim, int block_size)\n{\n    for (int t = 0; t < num_tokens; t++) {\n"
        "        const int64_t slot = slot_mapping[t];\n        if (slot < 0)\n            continue;",
        "int num_kv_heads, int head_dim, int block_size)\n{\n    for (int t = 0; t < num_tokens; t++) {\n"
        "        const int64_t slot = slot_mapping[t];\n        if (slot < 0)\n            break;"),
    "slot_offset": ("slots[i] = (int64_t)table[pos / block_size] * block_size + pos % block_size;",
                    "slots[i] = (int64_t)table[pos / block_size] * block_size + (pos + 1) % block_size;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_mutant_fails_a_pin(name, tmp_path):
    before, after = MUTATIONS[name]
    with open(oracle.SOURCE) as f:
        src = f.read()
    assert before in src, f"mutation site for {name} not found"
    mutated = src.replace(before, after)
    path = os.path.join(tmp_path, "mutant.c")
    with open(path, "w") as f:
        f.write(mutated)
    lib = oracle.build(path, os.path.join(tmp_path, "libmutant.so"), force=True)
    orc = oracle.Oracle(lib)
    failed = []
    for pin in oracle_pins.ALL_PINS:
        try:
            pin(orc)
        except AssertionError:
            failed.append(pin.__name__)
            break
    assert failed, f"mutant {name} passed every pin"
