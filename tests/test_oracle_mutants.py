"""Planted-mistake tests for the oracle's pins (CPU only).

Each mutant is a copy of ``oracle/pa_oracle.c`` with one plausible mistake (a wrong
index, a dropped term, a swapped operand, a wrong constant), compiled into a
temporary library.  The pin checks of ``test_oracle_pins.py`` run against it in a
subprocess (a mutant that reads out of bounds may crash, which also counts as
caught); at least one check must fail for every mutant.
"""
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "gqa_head_map": ("const int h = hq / G;", "const int h = hq % J->num_kv_heads;"),
    "q_uses_kv_head": ("const int64_t qo = (((int64_t)i * T + tq) * J->num_q_heads + hq) * D;",
                       "const int64_t qo = (((int64_t)i * T + tq) * J->num_q_heads + hq / G) * D;"),
    "q_token_index": ("const int64_t qo = (((int64_t)i * T + tq) * J->num_q_heads + hq) * D;",
                      "const int64_t qo = (((int64_t)i * T) * J->num_q_heads + hq) * D;"),
    "causal_off_by_one": ("const int n = L - T + tq + 1;", "const int n = L - T + tq;"),
    "causal_ignored": ("const int n = L - T + tq + 1;", "const int n = L;"),
    "causal_reversed": ("const int n = L - T + tq + 1;", "const int n = L - tq;"),
    "table_index_mod": ("int64_t phys = table[t / block_size];", "int64_t phys = table[t % block_size];"),
    "token_in_block_div": ("(int64_t)(t % block_size) * num_kv_heads * head_dim",
                           "(int64_t)(t / block_size) * num_kv_heads * head_dim"),
    "head_stride": ("(int64_t)h * head_dim + d;", "(int64_t)h * block_size + d;"),
    "no_scale": ("        s *= J->scale;\n", "\n"),
    "drop_last_token": ("      for (int t = 0; t < n; ++t) {\n        double w",
                        "      for (int t = 0; t + 1 < n; ++t) {\n        double w"),
    "no_normalisation": ("for (int d = 0; d < D; ++d) o[d] /= z;", ""),
    "k_from_v_cache": ("load_elem(J->k_cache, kv_offset", "load_elem(J->v_cache, kv_offset"),
    "no_max_shift": ("double w = exp(scores[t] - m);", "double w = exp(scores[t]);"),
    "q_element_index": ("load_elem(J->q, qo + d, J->q_dtype)", "load_elem(J->q, qo, J->q_dtype)"),
    "f16_bias": ("ldexp((double)(m + 1024), e - 25)", "ldexp((double)(m + 1024), e - 24)"),
    "f16_subnormal": ("v = ldexp((double)m, -24);", "v = ldexp((double)m, -25);"),
    "f16_hidden_bit": ("ldexp((double)(m + 1024), e - 25)", "ldexp((double)(m + 512), e - 25)"),
    "bf16_shift": ("uint32_t u = (uint32_t)b << 16;", "uint32_t u = (uint32_t)b << 15;"),
    "reshape_block_pos_swapped": ("int64_t blk = s / block_size, pos = s % block_size;",
                                  "int64_t blk = s % block_size, pos = s / block_size;", 0),
    "reshape_negative_slot_written": ("if (s < 0) continue;", "if (s < 0) s = 0;", 0),
    "e4m3_store_block_pos_swapped": ("int64_t blk = s / block_size, pos = s % block_size;",
                                     "int64_t blk = s % block_size, pos = s / block_size;", 1),
    "e4m3_store_negative_slot_written": ("if (s < 0) continue;", "if (s < 0) s = 0;", 1),
    "reshape_ignores_head": ("k + (t * k_token_stride + (int64_t)h * head_dim) * elem_bytes",
                             "k + (t * k_token_stride) * elem_bytes"),
    "copy_direction": ("memmove(k_cache + dst * block_bytes, k_cache + src * block_bytes",
                       "memmove(k_cache + src * block_bytes, k_cache + dst * block_bytes"),
    "e4m3_bias": ("else v = ldexp((double)(8 + m), e - 10);", "else v = ldexp((double)(8 + m), e - 9);"),
    "e4m3_nan_rule": ("if (e == 15 && m == 7) return NAN;", "if (e == 15) return NAN;"),
    "e4m3_truncates": ("int q = (int)rint(a / ldexp(1.0, E - 1 - 3));", "int q = (int)floor(a / ldexp(1.0, E - 1 - 3));"),
    "e4m3_no_saturation": ("if (a > 448.0) return sign | 0x7e;", "if (a > 448.0) return sign | 0x7f;"),
    "e4m3_subnormal_quantum": ("code = (int)rint(a / ldexp(1.0, -9));", "code = (int)rint(a / ldexp(1.0, -10));"),
    "e4m3_store_multiplies": ("float qk = xk / k_scale;", "float qk = xk * k_scale;"),
    "e4m3_k_scale_dropped": ("if (J->kv_dtype == OR_E4M3) s *= J->k_scale;", ""),
    "e4m3_v_scale_dropped": ("for (int d = 0; d < D; ++d) o[d] *= J->v_scale;", ";"),
    "swap_direction": ("memcpy(dst_k + d * block_bytes, src_k + s * block_bytes, (size_t)block_bytes);",
                       "memcpy(dst_k + s * block_bytes, src_k + d * block_bytes, (size_t)block_bytes);"),
    "swap_skips_v": ("    memcpy(dst_v + d * block_bytes, src_v + s * block_bytes, (size_t)block_bytes);\n", ""),
    "copy_skips_v": ("    memmove(v_cache + dst * block_bytes, v_cache + src * block_bytes, (size_t)block_bytes);\n",
                     ""),
}

RUNNER = r"""
import sys
sys.path.insert(0, {root!r})
import oracle
from tests import test_oracle_pins as P
lib = oracle._load({lib!r})
failed = []
for check in P.ALL_CHECKS:
    try:
        check(lib)
    except Exception as e:  # AssertionError, OracleError, ...
        failed.append(check.__name__)
print("FAILED:" + ",".join(failed))
sys.exit(1 if failed else 0)
"""


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    find, repl, *which = MUTANTS[name]
    src = open(SRC, encoding="utf-8").read()
    if which:  # the pattern occurs more than once: mutate the given occurrence only
        idx = -1
        for _ in range(which[0] + 1):
            idx = src.index(find, idx + 1)
        mutated = src[:idx] + repl + src[idx + len(find):]
    else:
        assert src.count(find) == 1, f"mutant {name}: pattern must occur exactly once"
        mutated = src.replace(find, repl)
    mutant_c = tmp_path / f"{name}.c"
    mutant_c.write_text(mutated, encoding="utf-8")
    lib = tmp_path / f"{name}.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-D_GNU_SOURCE",
                    str(mutant_c), "-o", str(lib), "-lm"], check=True)
    r = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=str(lib))],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode != 0, f"mutant {name} survived every pin:\n{r.stdout}\n{r.stderr[-2000:]}"


def test_runner_passes_unmodified_oracle(tmp_path):
    """The same runner on the real oracle source must report no failure."""
    lib = tmp_path / "clean.so"
    subprocess.run(["gcc", "-std=c11", "-O2", "-fPIC", "-shared", "-pthread", "-D_GNU_SOURCE",
                    SRC, "-o", str(lib), "-lm"], check=True)
    r = subprocess.run([sys.executable, "-c", RUNNER.format(root=ROOT, lib=str(lib))],
                       capture_output=True, text=True, timeout=300, cwd=ROOT)
    assert r.returncode == 0, r.stdout + r.stderr[-2000:]
