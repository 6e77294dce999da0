"""Mutation check of the oracle pins.

Each case plants one plausible mistake in a private copy of the oracle's C
source (never in the committed file), builds it, and runs the pin suite in
tests/test_oracle.py against the broken library.  The pins must catch every
mistake: a dropped scale, a swapped nibble, a wrong exponent bias, a wrong
head map, an off-by-one causal limit, a transposed cache index, a flipped
softmax sign, a wrong combine weight, a wrong fold direction; and in the
cache writer a wrong position, a swapped nibble, truncation instead of
rounding, a wrong INT8 range, ties to the odd e4m3 code and a quotient
taken as x times a rounded 1 / s instead of one correctly rounded division.
"""
import os
import shutil
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ORACLE_DIR = os.path.join(ROOT, "oracle")

MUTANTS = {
    "nibble_order": ("(d % 2 == 0) ? (byte & 0xF) : (byte >> 4)",
                     "(d % 2 == 1) ? (byte & 0xF) : (byte >> 4)"),
    "int4_unsigned": ("nib >= 8 ? nib - 16 : nib", "nib"),
    "e4m3_bias": ("e - 7)", "e - 8)"),
    "e4m3_subnormal": ("1 - 7)", "0 - 7)"),
    "gqa_head_map": ("const int kv = h / G; /* reading",
                     "const int kv = h % p->kv_num_heads; /* reading"),
    "causal_off_by_one": ("(Lb - qb) + i + 1", "(Lb - qb) + i"),
    "drop_k_scale": ("acc += qrow[d] * (k_scale[kv * D + d] * oracle_decode(p->kv_dtype, krow, d));",
                     "acc += qrow[d] * oracle_decode(p->kv_dtype, krow, d);"),
    "drop_v_scale": ("orow[d] += w * (v_scale[kv * D + d] * oracle_decode(p->kv_dtype, vrow, d));",
                     "orow[d] += w * oracle_decode(p->kv_dtype, vrow, d);"),
    "softmax_sign": ("s[t] = exp(s[t] - smax);", "s[t] = exp(smax - s[t]);"),
    "slot_shift": ("int slot = t % p->block_size;", "int slot = (t + 1) % p->block_size;"),
    "cache_index_transposed": ("((int64_t)phys * p->block_size + slot) * p->kv_num_heads + kv",
                               "((int64_t)phys * p->kv_num_heads + kv) * p->block_size + slot"),
    "combine_weight": ("const double w = exp(lse_parts[sp * rows + r] - lse);",
                       "const double w = exp(lse_parts[sp * rows + r] - mx);"),
    "fold_direction": ("ldexp(k_scale[kv * D + d], -e)", "ldexp(k_scale[kv * D + d], e)"),
    "default_scale": ("1.0 / sqrt((double)p->head_size)", "1.0 / (double)p->head_size"),
    "append_position": ("const int t = (Lb - qb) + i;", "const int t = i;"),
    "append_nibble": ("if (d % 2 == 0)\n      row[d / 2] = (uint8_t)((row[d / 2] & 0xF0) | nib);",
                      "if (d % 2 == 1)\n      row[d / 2] = (uint8_t)((row[d / 2] & 0xF0) | nib);"),
    "quantise_truncates": ("const float r = rintf(q);", "const float r = truncf(q);"),
    "quantise_int8_range": ("? -8 : -127;", "? -8 : -128;"),
    "e4m3_tie_odd": ("(d == best_d && (c & 1) == 0)", "(d == best_d && (c & 1) == 1)"),
    "quantise_inverse_multiply": ("const float q = x / s;", "const float q = x * (1.0f / s);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_mutant(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(os.path.join(ORACLE_DIR, "oracle.c")).read()
    assert old in src, "mutation anchor vanished from oracle.c: %r" % old
    mutated = src.replace(old, new, 1)
    shutil.copy(os.path.join(ORACLE_DIR, "oracle.h"), tmp_path / "oracle.h")
    (tmp_path / "oracle.c").write_text(mutated)
    lib = str(tmp_path / "libmutant.so")
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-o", lib,
                           str(tmp_path / "oracle.c"), "-lm"])
    env = dict(os.environ, ORACLE_LIB=lib)
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider",
                        os.path.join(ROOT, "tests", "test_oracle.py")], cwd=ROOT, env=env,
                       capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, "pins did not catch mutant %s:\n%s" % (name, r.stdout[-2000:])
