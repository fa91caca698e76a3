"""The oracle's pins must catch plausible mistakes.

Each case plants one mistake in a copy of the oracle's C source (on the CPU,
in a temporary directory), builds it, and runs the oracle pin tests against
that build in a subprocess.  The pins pass on the real oracle; every planted
mistake must make at least one of them fail.
"""
import os
import subprocess
import sys

import pytest

import oracle

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "oracle.c")

MUTANTS = {
    "decode_bias_8": ("v = ldexp(1.0 + (double)m / 8.0, e - 7);",
                      "v = ldexp(1.0 + (double)m / 8.0, e - 8);"),
    "ties_away_from_zero": ("((k + 1) & 1) == 0", "1"),
    "overflow_to_nan": ("if (a > 448.0)\n        return sign | 0x7Eu;", "if (a > 448.0)\n        return sign | 0x7Fu;"),
    "reciprocal_multiply": ("volatile float y = x / scale;", "volatile float y = x * (1.0f / scale);"),
    "dropped_sm_scale": ("scores[t] = (double)sm_scale * dot;", "scores[t] = dot;"),
    "wrong_kv_head": ("int32_t hk = item % num_kv_heads;", "int32_t hk = (item + 1) % num_kv_heads;"),
    "lse_log2": ("double lse_v = m + log(sum);", "double lse_v = m + log2(sum);"),
    "tag_check_skips_last_entry": ("for (int32_t j = 0; j < used; ++j) {\n                int32_t pid = page_table[(int64_t)b * max_pages + j];\n                if (pid < 0 || pid >= num_pages) {",
                                   "for (int32_t j = 0; j < used - 1; ++j) {\n                int32_t pid = page_table[(int64_t)b * max_pages + j];\n                if (pid < 0 || pid >= num_pages) {"),
    "append_slot_off_by_one": ("int32_t pos = L - 1;\n        int32_t pid = page_table[(int64_t)b * max_pages + pos / page_size];\n        if (pid < 0 || pid >= num_pages)\n            continue;\n        int32_t slot = pos % page_size;\n        for (int32_t h = 0; h < num_kv_heads; ++h) {\n            for (int32_t d = 0; d < head_dim; ++d) {\n                int64_t src = ((int64_t)b * num_kv_heads + h) * head_dim + d;\n                int64_t dst = (((int64_t)pid * num_kv_heads + h) * page_size + slot) * head_dim + d;\n                k_cache[dst] = orc_quantize_bf16",
                               "int32_t pos = L - 1;\n        int32_t pid = page_table[(int64_t)b * max_pages + pos / page_size];\n        if (pid < 0 || pid >= num_pages)\n            continue;\n        int32_t slot = (pos + 1) % page_size;\n        for (int32_t h = 0; h < num_kv_heads; ++h) {\n            for (int32_t d = 0; d < head_dim; ++d) {\n                int64_t src = ((int64_t)b * num_kv_heads + h) * head_dim + d;\n                int64_t dst = (((int64_t)pid * num_kv_heads + h) * page_size + slot) * head_dim + d;\n                k_cache[dst] = orc_quantize_bf16"),
    "int4_nibble_order": ("int32_t bit = (m % 2 == 0) ? 4 * (m / 2) : 16 + 4 * (m / 2);",
                          "int32_t bit = 4 * m;"),
    "int4_word_big_endian": ("uint32_t word = (uint32_t)w_tiles[at] | ((uint32_t)w_tiles[at + 1] << 8) |",
                             "uint32_t word = ((uint32_t)w_tiles[at] << 24) | ((uint32_t)w_tiles[at + 1] << 8) |"),
    "int4_unsigned_codes": ("return nibble >= 8 ? nibble - 16 : nibble;", "return nibble;"),
    "int4_tile_transposed": ("int64_t at = tile * 16384 + (int64_t)(j % 128) * 128 + (int64_t)((i % 256) / 8) * 4;",
                             "int64_t at = tile * 16384 + (int64_t)((i % 256) / 8) * 512 + (j % 128) * 4;"),
    "int4_scale_group_major": ("int64_t at = ((int64_t)(j / 128) * (k / group) + i / group) * 128 + j % 128;",
                               "int64_t at = (int64_t)j * (k / group) + i / group;"),
    "int4_group_off_by_one": ("int64_t at = ((int64_t)(j / 128) * (k / group) + i / group) * 128 + j % 128;",
                              "int64_t at = ((int64_t)(j / 128) * (k / group) + (i + 1) % k / group) * 128 + j % 128;"),
    "merge_l_unweighted": ("lsum += l[s] * w;", "lsum += l[s];"),
    "merge_o_unweighted": ("out[d] += o[(int64_t)s * head_dim + d] * w;",
                           "out[d] += o[(int64_t)s * head_dim + d];"),
    "partial_not_shifted_by_max": ("double w = exp(scores[t - t0] - m);\n        l += w;",
                                   "double w = exp(scores[t - t0]);\n        l += w;"),
    "transposed_v_index": ("o[d] += w * kv_element(kv_dtype, v_cache, (double)v_scale, pid,\n                                           num_kv_heads, hk, page_size, t % page_size,\n                                           head_dim, d);",
                           "o[d] += w * kv_element(kv_dtype, v_cache, (double)v_scale, pid,\n                                           num_kv_heads, hk, page_size, d % page_size,\n                                           head_dim, t % head_dim);"),
}


@pytest.mark.slow
@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    before, after = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(before) == 1, f"mutation anchor for {name} not unique"
    mutated = tmp_path / "oracle_mutant.c"
    mutated.write_text(src.replace(before, after))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", *oracle.CFLAGS, str(mutated), "-o", str(lib), "-lm"], check=True,
                   capture_output=True)
    env = dict(os.environ, PAGEDKV_ORACLE_LIB=str(lib))
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_codec.py"),
                        os.path.join(ROOT, "tests", "test_oracle_paths.py"),
                        os.path.join(ROOT, "tests", "test_oracle_int4.py"),
                        os.path.join(ROOT, "tests", "test_oracle_merge.py")],
                       env=env, cwd=ROOT, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"planted mistake {name} passed every pin:\n{r.stdout[-2000:]}"
