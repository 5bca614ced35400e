"""The oracle's pins must catch plausible mistakes (CPU only).

Each case plants one mistake in a copy of the oracle's C source (a dropped term,
a wrong index, a transposed operand, a wrong rounding rule), builds it, and runs
the oracle pin suites against that build in a child process.  The child must
fail; a mutant that passes every pin would mean the pins do not pin.  The
mutants build and run concurrently.
"""

import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "offset_from_quotient": ("int64_t off = l % block_size;", "int64_t off = (l / block_size) % block_size;"),
    "block_from_position": ("int64_t phys = table[l / block_size];", "int64_t phys = table[0];"),
    "scale_dropped": ("    s *= scale;\n", "\n"),
    "no_max_shift": ("double p = exp(scratch[j - lo] - m);", "double p = exp(scratch[j - lo]);"),
    "gqa_interleaved": ("int h = kvh * group + g;\n        int64_t qrow", "int h = g * num_kv_heads + kvh;\n        int64_t qrow"),
    "kv_swapped": ("acc += scratch[j - lo] * V[", "acc += scratch[j - lo] * K["),
    "slot_offset_swapped": ("int64_t b = s / block_size, o = s % block_size;", "int64_t o = s / block_size, b = s % block_size;"),
    "fp8_scale_multiplied": ("float yk = xk / k_scale;", "float yk = xk * k_scale;"),
    "e4m3_ties_odd": ("c = (lo & 1) ? hi : lo;", "c = (lo & 1) ? lo : hi;"),
    "e4m3_bias_off": ("v = ldexp((double)(8 + m), e - 10);", "v = ldexp((double)(8 + m), e - 11);"),
    "merge_unweighted": ("double w = lp * exp(m[r * max_parts + p] - M);", "double w = exp(m[r * max_parts + p] - M);"),
    "f16_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "dequant_scale_dropped": ("        k *= k_scale;\n", "\n"),
    "swap_wrong_pool": ("(const char*)src_key_caches[l] + src * block_bytes", "(const char*)dst_key_caches[l] + src * block_bytes"),
    "blocks_of_16": ("int64_t phys = table[l / block_size];\n    int64_t off = l % block_size;",
                     "int64_t phys = table[l / 16];\n    int64_t off = l % 16;"),
    "prefill_position_off_by_one": ("int pos = L - nq + j; /* this query token's position */",
                                    "int pos = L - nq + j - 1; /* this query token's position */"),
    "prefill_gqa_interleaved": ("int h = kvh * group + g;\n          int64_t row = ((int64_t)(q0 + j)",
                                "int h = g * num_kv_heads + kvh;\n          int64_t row = ((int64_t)(q0 + j)"),
    "prefill_not_causal": ("attend_rows(out + row, NULL, NULL, q, K, V, 0, pos + 1, head_dim, scale, sc);", "attend_rows(out + row, NULL, NULL, q, K, V, 0, L, head_dim, scale, sc);"),
    "copy_wrong_direction": ("memcpy((char*)key_caches[l] + dst * block_bytes, (char*)key_caches[l] + src * block_bytes,",
                             "memcpy((char*)key_caches[l] + src * block_bytes, (char*)key_caches[l] + dst * block_bytes,"),
    "partition_overlap": ("int lo = p * partition_size, hi = lo + partition_size;",
                          "int lo = p * partition_size, hi = lo + partition_size + 1;"),
    "reshape_value_from_key": ("memcpy((char*)value_cache + dst_row * ec, (const char*)value + src_row * es,",
                               "memcpy((char*)value_cache + dst_row * ec, (const char*)key + src_row * es,"),
    "bf16_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "merge_not_normalised": ("    for (int d = 0; d < head_dim; ++d) out[r * head_dim + d] /= W;\n", "\n"),
    "decode_newest_token_dropped": (
        "attend_rows(out + qrow, NULL, NULL, q, K, V, 0, L, head_dim, scale, sc);",
        "attend_rows(out + qrow, NULL, NULL, q, K, V, 0, L - 1, head_dim, scale, sc);"),
    "e4m3_saturates_to_nan": ("if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
                              "if (a >= 448.0) return (uint8_t)(sign | 0x7F);"),
    "dequant_v_by_k_scale": ("        v *= v_scale;\n", "        v *= k_scale;\n"),
    "quant_v_by_k_scale": ("float yv = xv / v_scale;", "float yv = xv / k_scale;"),
    "f16_normal_bias": ("v = ldexp((double)(1024 + m), e - 25);", "v = ldexp((double)(1024 + m), e - 24);"),
    "e4m3_subnormal_scale": ("v = ldexp((double)m, -9);", "v = ldexp((double)m, -10);"),
    "partition_last_short": ("if (hi > L) hi = L;", "if (hi > L) hi = L - 1;"),
    "copy_value_skipped": ("      memcpy((char*)value_caches[l] + dst * block_bytes,\n"
                           "             (char*)value_caches[l] + src * block_bytes, (size_t)block_bytes);\n",
                           ""),
    "copy_first_layer_only": ("    for (int l = 0; l < num_layers; ++l) {\n      memcpy((char*)key_caches[l]",
                              "    for (int l = 0; l < 1; ++l) {\n      memcpy((char*)key_caches[l]"),
    "swap_value_from_key": ("(const char*)src_value_caches[l] + src * block_bytes",
                            "(const char*)src_key_caches[l] + src * block_bytes"),
    "gather_kv_head_ignored": (
        "int64_t row = ((phys * num_kv_heads + kvh) * block_size + off) * (int64_t)head_dim;",
        "int64_t row = ((phys * num_kv_heads) * block_size + off) * (int64_t)head_dim;"),
    "reshape_token_major": (
        "int64_t dst_row = ((b * num_kv_heads + h) * block_size + o) * (int64_t)head_dim;",
        "int64_t dst_row = ((b * block_size + o) * num_kv_heads + h) * (int64_t)head_dim;"),
    "prefill_query_start_ignored": ("int64_t row = ((int64_t)(q0 + j) * num_heads + h) * head_dim;",
                                    "int64_t row = ((int64_t)j * num_heads + h) * head_dim;"),
    "partition_sum_lost": ("if (l_out) *l_out = sum;", "if (l_out) *l_out = 1.0;"),
    "e4m3_nan_saturates": ("if (isnan(y)) return 0x7F;", "if (isnan(y)) return 0x7E;"),
}


def _run_mutant(name):
    """Build the oracle with one planted mistake and run the pin suites on it in a
    child process; returns (the child's exit status, the end of its output)."""
    old, new = MUTANTS[name]
    src = open(SRC).read()
    if src.count(old) != 1:
        return None, f"mutation site for {name} not found exactly once"
    with tempfile.TemporaryDirectory() as tmp:
        csrc = os.path.join(tmp, "mutant.c")
        lib = os.path.join(tmp, "libmutant.so")
        with open(csrc, "w") as f:
            f.write(src.replace(old, new))
        subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-o", lib,
                        csrc, "-lm"], check=True)
        env = dict(os.environ, PA_ORACLE_LIB_OVERRIDE=lib, OMP_NUM_THREADS="2")
        r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                            os.path.join(ROOT, "tests", "test_oracle_formats.py"),
                            os.path.join(ROOT, "tests", "test_oracle_cache_ops.py"),
                            os.path.join(ROOT, "tests", "test_oracle_decode.py")],
                           cwd=ROOT, env=env, capture_output=True, text=True, timeout=900)
        return r.returncode, r.stdout[-2000:]


@pytest.fixture(scope="module")
def outcomes():
    """Every mutant's outcome; the mutants build and run concurrently."""
    workers = max(1, min(8, (os.cpu_count() or 2) // 2))
    with ThreadPoolExecutor(max_workers=workers) as ex:
        return dict(zip(MUTANTS, ex.map(_run_mutant, MUTANTS)))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, outcomes):
    rc, out = outcomes[name]
    assert rc is not None, out
    assert rc != 0, f"mutant {name} passed every pin:\n{out}"
