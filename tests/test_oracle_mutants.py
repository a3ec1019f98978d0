"""Plant one plausible mistake at a time in a copy of the oracle's C source
(on the CPU, in a temporary directory) and check that at least one pin
catches it.  This shows the pins constrain every step: causal bound, scale,
max subtraction, group mapping, score accumulation, tie order, window extent,
gate direction, and the own-window layer's buffer and row offset."""
import os
import shutil

import pytest

import oracle
import oracle_pins
from oracle import hsref

MUTANTS = {
    "causal_bound_off_by_one": ("const int n = pos + 1;\n            int *keys", "const int n = pos;\n            int *keys"),
    "no_scale": ("s[t] = scale * dot_fd(", "s[t] = dot_fd("),
    "prob_without_max": ("double p = exp(s[t] - m) / l;", "double p = exp(s[t]) / l;"),
    "group_mapping": ("const int h = g * G + hh;\n                    const float *q = q_rows",
                      "const int h = hh * Hkv + g;\n                    const float *q = q_rows"),
    "score_overwrite": ("if (acc_p) acc_p[t] += p;", "if (acc_p) acc_p[t] = p;"),
    "tie_to_higher_index": ("return (x->j > y->j) - (x->j < y->j);", "return (x->j < y->j) - (x->j > y->j);"),
    "window_one_wider": ("int lo = pos - window + 1;", "int lo = pos - window;"),
    "gate_swapped": ("out[o + c] = gs * og[c] + (1.0 - gs) * ol[c];",
                     "out[o + c] = gs * ol[c] + (1.0 - gs) * og[c];"),
    "lse_without_log": ("return m + log(l);", "return m + l;"),
    "topk_keeps_k_minus_1": ("int take = n < topk ? n : topk;", "int take = n < topk ? n : topk - 1;"),
    # the own-window layer's local branch reading the shared cache at the
    # buffer's row numbers (in range, wrong values)
    "own_window_reads_shared_cache": (
        "attend_list(q, kw, vw, b, g, Lwin, Hkv, d, scale, keys_l, nl, s, ol, NULL);",
        "attend_list(q, k, v, b, g, Lkv, Hkv, d, scale, keys_l, nl, s, ol, NULL);"),
    # the own-window buffer's first row taken one position too late (every
    # read stays inside the buffer: rows are validated before any is read)
    "own_window_offset_plus_one": ("const int woff = kw ? Lkv - Lwin : 0;",
                                   "const int woff = kw ? Lkv - Lwin + 1 : 0;"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_mutant_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = open(hsref._SRC).read()
    assert src.count(old) == 1, f"mutation site for {name} not unique/found"
    mut_src = tmp_path / "hsref_mut.c"
    mut_src.write_text(src.replace(old, new))
    lib = str(tmp_path / "libhsref_mut.so")
    hsref.build(force=True, src=str(mut_src), lib=lib)
    caught = []
    try:
        oracle.use_library(lib)
        for pin in oracle_pins.ALL_PINS:
            try:
                pin()
            except (AssertionError, ValueError):
                caught.append(pin.__name__)
    finally:
        oracle.use_library(None)
    assert caught, f"no pin caught mutant {name}"
