"""The oracle's pins must catch plausible slips.

Each case below plants one mistake in a private copy of oracle/pa_oracle.c
(on the CPU, in a temporary directory), builds it, and runs the pin suites
against that build; at least one pin must fail.  The committed oracle is
never modified.
"""
from __future__ import annotations

import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "pa_oracle.c")

MUTANTS = {
    "exp_sign_flipped": ("double w = exp(s[t] - m);", "double w = exp(m - s[t]);"),
    "normalisation_dropped": ("o[d] /= Z;", "o[d] /= 1.0;"),
    "scale_dropped": ("s[t] = scale * acc;", "s[t] = acc;"),
    "row_head_mapping_modulo": ("const int b = rows_b[i], h = rows_h[i], kvh = h / G;",
                                "const int b = rows_b[i], h = rows_h[i], kvh = h % Hkv;"),
    # first occurrence: the grouped-head loop of oracle_paged_decode
    "group_heads_interleaved": ("const int h = kvh * G + g;", "const int h = g * Hkv + kvh;"),
    "in_block_offset_reversed": ("int64_t offset = t % block_size;", "int64_t offset = block_size - 1 - t % block_size;"),
    "pool_layout_transposed": ("int64_t row = ((phys * Hkv + kvh) * block_size + offset) * D;",
                               "int64_t row = ((phys * block_size + offset) * Hkv + kvh) * D;"),
    "value_read_from_key_pool": ("Vc[t * D + d] = widen(v_pool, row + d, dtype);", "Vc[t * D + d] = widen(k_pool, row + d, dtype);"),
    "slot_offset_wrong": ("slots[i] = phys * block_size + pos % block_size;", "slots[i] = phys * block_size + pos / block_size;"),
    "cache_write_value_from_key": ("memcpy((char*)v_pool + dst * row_bytes, (const char*)value + src * row_bytes, row_bytes);",
                                   "memcpy((char*)v_pool + dst * row_bytes, (const char*)key + src * row_bytes, row_bytes);"),
    "copy_blocks_skips_v": ("memmove((char*)v_pool + dst * block_bytes, (const char*)v_pool + src * block_bytes, block_bytes);", ""),
    "bf16_rounds_one_bit_short": ("int qexp = e - 8;", "int qexp = e - 7;"),
    "prefill_causal_excludes_self": ("bad |= attend(qrow, Kc, Vc, pos + 1, D,", "bad |= attend(qrow, Kc, Vc, pos, D,"),
    "prefill_causal_sees_one_ahead": ("bad |= attend(qrow, Kc, Vc, pos + 1, D,", "bad |= attend(qrow, Kc, Vc, pos + 2 > L ? L : pos + 2, D,"),
    "prefill_query_position_from_start": ("const int64_t pos = L - n + i;", "const int64_t pos = i;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(name, tmp_path):
    old, new = MUTANTS[name]
    text = open(SRC).read()
    assert text.count(old) >= 1, f"mutation site for {name} not found"
    mutant = tmp_path / "pa_oracle_mutant.c"
    mutant.write_text(text.replace(old, new, 1))
    lib = tmp_path / "liboracle_mutant.so"
    subprocess.run(["gcc", "-O2", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", str(lib),
                    str(mutant), "-lm"], check=True)
    env = dict(os.environ, PA_ORACLE_LIB=str(lib), OMP_NUM_THREADS="2")
    pins = [os.path.join(ROOT, "tests", f) for f in ("test_oracle_pins.py", "test_oracle_cache_ops.py",
                                                      "test_oracle_prefill.py")]
    r = subprocess.run([sys.executable, "-m", "pytest", "-x", "-q", "-p", "no:cacheprovider", *pins],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode != 0, f"mutant {name} survived the pins:\n{r.stdout[-2000:]}"
