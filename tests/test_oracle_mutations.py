"""Each plausible mistake planted in a copy of the oracle must fail a pin.

The mistakes are planted in a temporary copy of ``oracle/pkv_oracle.c`` on the
CPU; the committed oracle is never modified.  This shows the pins in
``oracle_checks.py`` can tell a correct oracle from a wrong one.
"""
import os
import subprocess

import pytest

import oracle
import oracle_checks as oc

SRC = os.path.join(os.path.dirname(oracle.__file__), "pkv_oracle.c")

MUTATIONS = {
    "gqa_map_modulo": ("int64_t g = head / group;", "int64_t g = head % num_kv_heads;"),
    "scale_dropped": ("z[i] = scale * dot;", "z[i] = dot;"),
    "block_index_swapped": ("int64_t block = table_row[pos / block_size];",
                            "int64_t block = table_row[pos % block_size];"),
    "last_position_dropped": ("int64_t n = p_end > p_begin ? p_end - p_begin : 0;",
                              "int64_t n = p_end > p_begin + 1 ? p_end - p_begin - 1 : 0;"),
    "values_read_from_keys": ("if (gather_row(v_cache,", "if (gather_row(k_cache,"),
    "half_exponent_bias": ("exp - 25);", "exp - 24);"),
    "append_token_head_transposed": ("const uint16_t *src = new_kv + (t * kv_heads + h) * head_dim;",
                                     "const uint16_t *src = new_kv + (h * num_tokens + t) * head_dim;"),
    "merge_weight_dropped": ("total += l[j] * w;", "total += l[j];"),
    "not_normalised": ("o[d] = o[d] / l;", "o[d] = o[d];"),
    "max_not_subtracted_sign": ("double w = exp(z[i] - m);", "double w = exp(m - z[i]);"),
    "copy_blocks_swapped": ("memmove(cache + dst * block_elems, cache + src * block_elems,",
                            "memmove(cache + src * block_elems, cache + dst * block_elems,"),
    "prefill_window_off_by_one": ("int64_t window = ctx - n + i + 1;", "int64_t window = ctx - n + i;"),
    "e4m3_bias": ("v = ldexp(1.0 + m / 8.0, e - 7);", "v = ldexp(1.0 + m / 8.0, e - 8);"),
    "e4m3_ties_odd": ("(err == best_err && (c & 1) == 0 && (best & 1) == 1)",
                      "(err == best_err && (c & 1) == 1 && (best & 1) == 0)"),
    "e4m3_scale_range": ("return amax > 0.0f ? amax / 448.0f : 1.0f;", "return amax > 0.0f ? amax / 240.0f : 1.0f;"),
    "e4m3_gather_block_swapped": ("int64_t phys = table_row[pos / block_size];",
                                  "int64_t phys = table_row[pos % block_size];"),
    "e4m3_append_head_transposed": ("const uint16_t *xrow = new_kv + (t * kv_heads + h) * head_dim;",
                                    "const uint16_t *xrow = new_kv + (h * num_tokens + t) * head_dim;"),
    "slot_mask_last_position_dropped": ("for (int64_t p = 0; p < lens[s]; ++p) {",
                                        "for (int64_t p = 0; p + 1 < lens[s]; ++p) {"),
    "slot_mask_whole_blocks": ("mask[b * block_size + p % block_size] = 1;",
                               "for (int64_t r = 0; r < block_size; ++r) mask[b * block_size + r] = 1;"),
    "slot_mask_row_from_block": ("mask[b * block_size + p % block_size] = 1;",
                                 "mask[b * block_size + p / block_size] = 1;"),
    "kv_sizing_factor": ("return 2 * seq_len * kv_heads * head_dim * dtype_bytes;",
                         "return seq_len * kv_heads * head_dim * dtype_bytes;"),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(tmp_path, name):
    old, new = MUTATIONS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation anchor not unique: {old!r}"
    path = tmp_path / "mutant.c"
    path.write_text(src.replace(old, new))
    so = str(tmp_path / "libmutant.so")
    subprocess.run(["gcc", "-O1", "-std=c11", "-fPIC", "-shared", "-fopenmp", str(path), "-o", so, "-lm"],
                   check=True)
    lib = oracle.load(so)
    caught = []
    for check in oc.ALL_CHECKS:
        try:
            check(lib)
        except (AssertionError, ValueError):
            caught.append(check.__name__)
    assert caught, f"no pin caught the planted mistake {name}"
