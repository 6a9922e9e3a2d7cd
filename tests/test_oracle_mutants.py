"""Mutation check of the oracle's pins.

Each mutant is a copy of oracle/moe_oracle.c with one plausible mistake planted
(a sign, a swapped operand, a tie-break, a nibble order, a transposed index, a
dropped term).  The mutant is compiled to a temporary library on the CPU and the
pin suite is run against it; every mutant must make some pin fail.
"""
import os
import subprocess
import sys
import tempfile
from concurrent.futures import ThreadPoolExecutor

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "moe_oracle.c")

MUTANTS = {
    "silu_sign": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = g / (1.0 + exp(g)) * u;"),
    "gate_up_swapped": ("h[n] = g / (1.0 + exp(-g)) * u;", "h[n] = u / (1.0 + exp(-u)) * g;"),
    "tie_to_higher_id": ("if (best < 0 || z[e] > z[best]) best = e;",
                         "if (best < 0 || z[e] >= z[best]) best = e;"),
    "nibble_order": ("int u = (k % 2 == 0) ? (byte & 15) : (byte >> 4);",
                     "int u = (k % 2 == 0) ? (byte >> 4) : (byte & 15);"),
    "scale_transposed": ("s[(size_t)(k / 128) * rows + row]", "s[(size_t)row * (K / 128) + k / 128]"),
    "combine_drops_sum": ("for (int c = 0; c < H; ++c) o[c] += wj * y[c];",
                          "for (int c = 0; c < H; ++c) o[c] = wj * y[c];"),
    "weights_unnormalised": ("w[(size_t)t * k + j] = exp((double)z[idx[(size_t)t * k + j]] - m) / den;",
                             "w[(size_t)t * k + j] = exp((double)z[idx[(size_t)t * k + j]] - m);"),
    "permute_unstable": ("for (int t = 0; t < T; ++t) {\n    for (int j = 0; j < k; ++j) {\n      size_t p",
                         "for (int t = T - 1; t >= 0; --t) {\n    for (int j = 0; j < k; ++j) {\n      size_t p"),
    "quant_floor": ("double rq = (quot < 0) ? -round_half_even(-(double)quot)\n"
                    "                                 : round_half_even((double)quot);",
                    "double rq = floor((double)quot);"),
    "fp16_ties_up": ("return fmod(fl, 2.0) == 0.0 ? fl : fl + 1.0;", "return fl + 1.0;"),
    "int8_unsigned": ("return (int)((const int8_t*)w)[(size_t)row * K + k];",
                      "return (int)((const uint8_t*)w)[(size_t)row * K + k];"),
    "down_scale_stride": ("load_row(ex->prec, ex->w2, ex->s2, H, I, m, row);",
                          "load_row(ex->prec, ex->w2, ex->s2, I, I, m, row);"),
    "dropped_last_k_column": ("for (int c = 0; c < H; ++c) g += x[c] * row[c];",
                              "for (int c = 0; c < H - 1; ++c) g += x[c] * row[c];"),
    "full_softmax_drops_first": ("for (int e = 0; e < E; ++e) den += exp((double)z[e] - m);",
                                 "for (int e = 1; e < E; ++e) den += exp((double)z[e] - m);"),
    "int8_q_128": ("const int Q = (prec == OR_INT4) ? 7 : 127;",
                   "const int Q = (prec == OR_INT4) ? 7 : 128;"),
    "fp16_subnormal_scale": ("v = ldexp((double)frac, -24);", "v = ldexp((double)frac, -25);"),
    "up_reads_gate_rows": ("load_row(ex->prec, ex->w13, ex->s13, 2 * I, H, I + n, row);",
                           "load_row(ex->prec, ex->w13, ex->s13, 2 * I, H, n, row);"),
    "cursor_not_advanced": ("int row = cursor[e]++;", "int row = cursor[e];"),
    "int4_offset_7": ("return u - 8;", "return u - 7;"),
    "topk_ascending": ("if (best < 0 || z[e] > z[best]) best = e;",
                       "if (best < 0 || z[e] < z[best]) best = e;"),
    "duplicate_ids_kept": ("if (idx[(size_t)t * k + jj] == e) return 1;",
                           "if (idx[(size_t)t * k + jj] == e + E) return 1;"),
    "layer_weight_slot": ("double wj = w[(size_t)t * k + j];\n          for (int c = 0; c < H; ++c) o[c] += wj * y[c];",
                          "double wj = w[(size_t)t * k + (j + 1) % k];\n          for (int c = 0; c < H; ++c) o[c] += wj * y[c];"),
    "router_transposed": ("oracle_bf16_to_double(wr[(size_t)e * H + c]);",
                          "oracle_bf16_to_double(wr[(size_t)c * E + e]);"),
    "router_drops_last_column": ("for (int c = 0; c < H; ++c)\n        acc +=",
                                 "for (int c = 0; c < H - 1; ++c)\n        acc +="),
    "combine_weight_slot": ("double wj = w[(size_t)t * k + j];\n      for (int c = 0; c < H; ++c) o[c] += wj * y_perm",
                            "double wj = w[(size_t)t * k + (j + 1) % k];\n      for (int c = 0; c < H; ++c) o[c] += wj * y_perm"),
}


def _run_mutant(name, tmp):
    old, new = MUTANTS[name]
    src = open(SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique"
    path = os.path.join(tmp, f"{name}.c")
    lib = os.path.join(tmp, f"lib{name}.so")
    open(path, "w").write(src.replace(old, new))
    subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", lib,
                           path, "-lm"])
    env = dict(os.environ, MOE_ORACLE_LIB=lib, OMP_NUM_THREADS="1")
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle_pins.py")],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    return name, r.returncode


def test_every_planted_mistake_fails_a_pin():
    with tempfile.TemporaryDirectory() as tmp:
        with ThreadPoolExecutor(max_workers=min(8, os.cpu_count() or 1)) as ex:
            results = dict(ex.map(lambda n: _run_mutant(n, tmp), MUTANTS))
    survivors = [n for n, rc in results.items() if rc == 0]
    assert not survivors, f"mutants not caught by any pin: {survivors}"
