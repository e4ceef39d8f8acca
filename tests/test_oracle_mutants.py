"""Planted mistakes in the oracle must be caught by the pins.

Each case copies ``oracle/bd_oracle.c`` with one plausible mistake swapped in
(a wrong mask bound, a transposed head mapping, a dropped term), compiles the
copy on the CPU, and requires at least one pin of ``pins.py`` to fail on it.
The real oracle source is never modified.
"""
import os
import subprocess

import pytest

import oracle
import pins

MUTANTS = {
    "obc_includes_own_block": ("return k_c < k_r; /* M_OBC",
                               "return k_c <= k_r; /* M_OBC"),
    "bc_excludes_own_block": ("return k_c <= k_r; /* M_BC",
                              "return k_c < k_r; /* M_BC"),
    "bd_sees_earlier_noisy": ("return k_c == k_r; /* M_BD",
                              "return k_c <= k_r; /* M_BD"),
    "clean_sees_noisy": ("return 0;              /* clean queries",
                         "return k_c == k_r;     /* clean queries"),
    "gqa_modulo_mapping": ("int g = h / group;", "int g = h % Hkv;"),
    "lse_drops_max": ("*lse = m + log(Z);", "*lse = log(Z);"),
    "scale_dropped": ("s[j] = scale * acc;", "s[j] = acc;"),
    "decode_causal_strict": ("(jc <= j)", "(jc < j)"),
    "decode_block_missing": ("if (c < cache_len + b) {", "if (c < cache_len) {"),
    "probs_unnormalised": ("out[t] += p * bf16", "out[t] += exp(s[j] - m) * bf16"),
    "combine_weight_wrong": ("double w = exp(lse_s[s] - *lse);",
                             "double w = exp(lse_s[s] - m);"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(oracle._SRC).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + old
    mutated = src.replace(old, new)
    cpath = os.path.join(tmp_path, "mut.c")
    spath = os.path.join(tmp_path, "libmut.so")
    with open(cpath, "w") as f:
        f.write(mutated)
    subprocess.run(["gcc", "-O1", "-std=c99", "-fopenmp", "-shared", "-fPIC",
                    "-o", spath, cpath, "-lm"], check=True)
    lib = oracle.load(spath)
    failed = []
    for pin in pins.ALL_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "no pin caught mutant " + name
