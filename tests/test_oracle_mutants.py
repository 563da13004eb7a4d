"""Plant plausible mistakes in copies of the oracle (CPU only) and check that the
pins catch every one.  The oracle source itself is never modified."""
import json
import os
import subprocess
import sys
import tempfile

import pytest

import oracle
import oracle_pins

# (name, text in pa_oracle.c, replacement).  Each must occur exactly once.
MUTANTS = [
    ("interleaved_gqa", "const int g = h / group;                       /* KV head of this query head */",
     "const int g = h % num_kv_heads;"),
    ("dropped_scale", "s[t] = scale * dot;\n    }\n\n    /* softmax", "s[t] = dot;\n    }\n\n    /* softmax"),
    ("sign_in_exponent", "s[t] = exp(s[t] - m);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)",
     "s[t] = exp(m - s[t]);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)"),
    ("min_for_max", "if (s[t] > m) m = s[t];\n    double z = 0.0;\n    for (int t = 0; t < L; ++t) {\n      s[t] = exp(s[t] - m);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)",
     "if (s[t] < m) m = s[t];\n    double z = 0.0;\n    for (int t = 0; t < L; ++t) {\n      s[t] = exp(s[t] - m);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)"),
    ("no_normalisation", "for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)", "for (int t = 0; t < L; ++t) s[t] = s[t];\n    if (weights)"),
    ("value_from_key_cache", '/* out = sum_t w_t * V_t, V_t gathered through the block table */\n    for (int t = 0; t < L; ++t) {\n      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];\n      int offset = t % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      for (int64_t d = 0; d < D; ++d) o[d] += s[t] * widen_one(v_cache, row + d, dtype);',
     '/* out = sum_t w_t * V_t, V_t gathered through the block table */\n    for (int t = 0; t < L; ++t) {\n      int32_t physical_block = block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];\n      int offset = t % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      for (int64_t d = 0; d < D; ++d) o[d] += s[t] * widen_one(k_cache, row + d, dtype);'),
    ("kv_head_zero", "int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      double dot",
     "int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + 0) * D;\n      double dot"),
    ("offset_off_by_one", "int offset = t % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      double dot",
     "int offset = (t + 1) % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      double dot"),
    ("block_index_by_offset", "block_tables[(int64_t)b * max_blocks_per_seq + t / block_size];\n      int offset = t % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      for",
     "block_tables[(int64_t)b * max_blocks_per_seq + t % 2];\n      int offset = t % block_size;\n      int64_t row = (((int64_t)physical_block * block_size + offset) * num_kv_heads + g) * D;\n      for"),
    ("transposed_slot_layout", "int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * row_bytes;",
     "int64_t dst = ((block * num_kv_heads + h) * block_size + offset) * row_bytes;"),
    ("bf16_shift", "uint32_t u = (uint32_t)h << 16;", "uint32_t u = (uint32_t)h << 15;"),
    ("fp16_bias", "v = ldexp((double)(1024 + frac), exp - 25);", "v = ldexp((double)(1024 + frac), exp - 24);"),
    ("fp16_subnormal", "v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    ("slot_rule_offset", "int64_t offset = pos % block_size;", "int64_t offset = (pos + 1) % block_size;"),
    ("copy_no_chain_check", "if ((j != i && block_mapping[2 * j + 1] == dst) || block_mapping[2 * j] == dst) {",
     "if ((j != i && block_mapping[2 * j + 1] == dst)) {"),
    ("copy_only_key_cache", "memcpy((char *)v_cache + dst * block_bytes, (const char *)v_cache + src * block_bytes, (size_t)block_bytes);",
     ""),
    ("negative_slot_written", "if (slot < 0) continue;\n    if (slot >= (int64_t)num_blocks * block_size) {\n      if (status == ORACLE_OK) status = ORACLE_BAD_SLOT;\n      continue;\n    }\n    int64_t block = slot / block_size;\n    int64_t offset = slot % block_size;\n    for (int h = 0; h < num_kv_heads; ++h) {\n      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * row_bytes;",
     "if (slot < 0) slot = 0;\n    if (slot >= (int64_t)num_blocks * block_size) {\n      if (status == ORACLE_OK) status = ORACLE_BAD_SLOT;\n      continue;\n    }\n    int64_t block = slot / block_size;\n    int64_t offset = slot % block_size;\n    for (int h = 0; h < num_kv_heads; ++h) {\n      int64_t dst = ((block * block_size + offset) * num_kv_heads + h) * row_bytes;"),
    ("weights_without_max_shift", "s[t] = exp(s[t] - m);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)",
     "s[t] = exp(s[t]);\n      z += s[t];\n    }\n    for (int t = 0; t < L; ++t) s[t] = s[t] / z;\n    if (weights)"),
    ("prefill_causal_off_by_one", "const int len = pos + 1;", "const int len = pos;"),
    ("prefill_no_offset", "const int pos = L - n + (int)(tok - query_start_loc[b]);",
     "const int pos = (int)(tok - query_start_loc[b]);"),
    ("e4m3_bias", "v = ldexp(8.0 + m, e - 10);", "v = ldexp(8.0 + m, e - 9);"),
    ("e4m3_ties_to_odd", "(d == best_d && (c & 1) == 0)", "(d == best_d && (c & 1) == 1)"),
    ("e4m3_no_saturation", "if (a >= 448.0) return (uint8_t)(sign ? 0xFE : 0x7E);", "if (a >= 1e30) return 0;"),
    ("e4m3_multiply_by_scale", "float q = x / scale;", "float q = x * scale;"),
    ("fp8_v_scale_dropped", "o[d] += s[t] * (e4m3_value(v_cache[row + d]) * v_scale);",
     "o[d] += s[t] * e4m3_value(v_cache[row + d]);"),
    ("fp8_write_k_with_v_scale", "k_cache[dst + d] = e4m3_encode((float)widen_one(key, src + d, dtype) / k_scale);",
     "k_cache[dst + d] = e4m3_encode((float)widen_one(key, src + d, dtype) / v_scale);"),
]


_RUNNER = """
import json, sys
sys.path[:0] = [{root!r}, {tests!r}]
import oracle, oracle_pins
o = oracle.Oracle({lib!r})
failed = []
for pin in oracle_pins.ALL_PINS:
    try:
        pin(o)
    except Exception as e:
        failed.append([pin.__name__, str(e)[:80]])
        break
print(json.dumps(failed))
"""


def _run_pins(lib):
    """Run every pin on a mutant library in a child process (a mutant may crash)."""
    here = os.path.dirname(os.path.abspath(__file__))
    code = _RUNNER.format(root=os.path.dirname(here), tests=here, lib=lib)
    env = dict(os.environ, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-c", code], capture_output=True, text=True, timeout=300, env=env)
    if r.returncode != 0:
        return [["crash", r.stderr[-200:]]]
    return json.loads(r.stdout.strip().splitlines()[-1])


def _check_mutant(name, old, new, workdir):
    src = open(oracle.SRC).read()
    if src.count(old) != 1:
        return name, [["anchor", "mutation anchor not found exactly once"]], False
    path = os.path.join(workdir, f"mutant_{name}.c")
    with open(path, "w") as f:
        f.write(src.replace(old, new))
    lib = oracle.compile_library(path, os.path.join(workdir, f"libmutant_{name}.so"), extra_flags=("-w",))
    return name, _run_pins(lib), True


@pytest.mark.slow
def test_every_mutant_is_caught():
    from concurrent.futures import ThreadPoolExecutor
    with tempfile.TemporaryDirectory() as d:
        with ThreadPoolExecutor(max_workers=max(2, min(8, os.cpu_count() or 2))) as ex:
            results = list(ex.map(lambda m: _check_mutant(*m, d), MUTANTS))
    bad = []
    for name, failed, anchored in results:
        if not anchored:
            bad.append(f"{name}: anchor missing")
        elif not failed:
            bad.append(f"{name}: passed every pin")
        else:
            print(f"{name}: caught by {failed[0][0]}")
    assert not bad, bad
