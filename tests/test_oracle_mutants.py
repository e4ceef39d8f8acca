"""Planted mistakes in the oracle must be caught by the pins.

Each case copies ``oracle/bd_oracle.c`` (or one of the oracle's numpy
modules) with one plausible mistake swapped in (a wrong mask bound, a
transposed head mapping, a dropped term), compiles or loads the copy on the
CPU, and requires at least one pin to fail on it.  The real oracle source is
never modified.
"""
import os
import subprocess
import types

import pytest

import oracle
import pins
import pins_ext
import pins_grad
from oracle import backward, cache_ops

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
    "mode2_sees_block": ("if (mode == 2)\n        return 0;",
                         "if (mode == 3)\n        return 0;"),
    "sprint_norm_first_head": ("for (h = 0; h < Hkv; ++h) {\n                const uint16_t *row",
                               "for (h = 0; h < 1; ++h) {\n                const uint16_t *row"),
    "sprint_ties_higher_first": ("return (x->p > y->p) - (x->p < y->p);",
                                 "return (x->p < y->p) - (x->p > y->p);"),
    "sprint_keep_floor": ("floor(r * (double)cnt + 0.5)", "floor(r * (double)cnt)"),
    "sprint_mean_over_capacity": ("mean /= n;", "mean /= S_cap;"),
    "sprint_conf_weight": ("(1.0 - alpha) * (double)conf", "alpha * (double)conf"),
}

PY_MUTANTS = {
    # module, old, new, pins
    "bwd_no_D": (backward, "dS = P * (dP - D)", "dS = P * dP"),
    "bwd_dk_no_scale": (backward, "dk = scale * (dS.T @ q)", "dk = dS.T @ q"),
    "bwd_dv_transposed": (backward, "dv = P.T @ dout", "dv = P @ dout"),
    "bwd_gqa_overwrite": (backward, "dk += bk", "dk = bk"),
    "bwd_D_axis": (backward, "D = (P * dP).sum(axis=1", "D = (P * dP).sum(axis=0"),
    "accept_counts_all": (cache_ops, "while j < b and draft[i, j] == target[i, j]:\n            j += 1",
                          "j = int((draft[i] == target[i]).sum())"),
    "append_keeps_len": (cache_ops, "lens[i] += n", "lens[i] += 0"),
    "crop_is_max": (cache_ops, "np.minimum(lens", "np.maximum(lens"),
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
    for pin in pins.ALL_PINS + pins_ext.EXT_PINS:
        try:
            pin(lib)
        except AssertionError:
            failed.append(pin.__name__)
    assert failed, "no pin caught mutant " + name


@pytest.mark.parametrize("name", sorted(PY_MUTANTS))
def test_py_mutant_is_caught(name):
    mod, old, new = PY_MUTANTS[name]
    src = open(mod.__file__).read()
    assert src.count(old) >= 1, "mutation anchor not found: " + old
    mut = types.ModuleType(mod.__name__ + "_mutant")
    mut.__file__ = mod.__file__
    exec(compile(src.replace(old, new), mod.__file__, "exec"), mut.__dict__)
    cands = pins_grad.GRAD_PINS if mod is backward else pins_ext.CACHE_PINS
    failed = []
    for pin in cands:
        try:
            pin(mut)
        except Exception:
            failed.append(pin.__name__)
    assert failed, "no pin caught mutant " + name
