"""Planted mistakes: every plausible slip in the oracle must fail at least one pin.

Each mutant is a copy of the oracle's C source with one edit (a dropped term, a wrong sign, an
off-by-one chunk boundary, a transposed or wrong index), compiled on the CPU into a temporary
library.  The pin battery from ``test_oracle_pins`` is then run against it with the mutant swapped
in; the test passes only if some pin fails.  The committed oracle itself is never modified.
"""
import os
import shutil
import subprocess
import tempfile

import numpy as np
import pytest

import oracle
import test_oracle_pins as pins

SRC = os.path.join(os.path.dirname(oracle.__file__), "wf_oracle.c")

# (name, text to find, replacement); every occurrence is replaced; all edits stay in bounds.
MUTANTS = [
    ("own_chunk_excluded", "jb->key_chunk[j] <= qc", "jb->key_chunk[j] < qc"),
    ("mask_reversed", "jb->key_chunk[j] <= qc", "jb->key_chunk[j] >= qc"),
    ("no_mask", "jb->key_chunk[j] <= qc", "jb->key_chunk[j] <= 1000000"),
    ("boundary_off_by_one", "t >= offsets[c] && t < offsets[c + 1]",
     "t >= offsets[c] && t <= offsets[c + 1]"),
    ("query_chunk_from_query_index", "jb->T_ctx + r", "r"),
    ("scale_dropped", "jb->scale * ", "1.0 * "),
    ("normalisation_dropped", "o_out[d] = (float)(acc[d] / den);", "o_out[d] = (float)(acc[d]);"),
    ("exp_sign_flipped", "s[j] = exp(s[j] - m);", "s[j] = exp(m - s[j]);"),
    ("key_head_wrong", "return jb->k + ((size_t)j * jb->H + h) * jb->D;",
     "return jb->k + ((size_t)j * jb->H + (h + 1) % jb->H) * jb->D;"),
    ("value_head_wrong", "return jb->v + ((size_t)j * jb->H + h) * jb->D;",
     "return jb->v + ((size_t)j * jb->H + 0) * jb->D;"),
    ("value_row_wrong", "value_row(jb, j, h)", "value_row(jb, T_kv - 1 - j, h)"),
    ("query_dim_transposed", "const double x = (double)qr[d];",
     "const double x = (double)qr[D - 1 - d];"),
    ("lse_max_dropped", "*lse_out = (float)(m + log(den));", "*lse_out = (float)(log(den));"),
]


def battery():
    yield "hand_cases", pins.test_hand_cases
    for s in range(4):
        yield f"brute_force[{s}]", lambda s=s: pins.test_brute_force_mask_matrix(s)
    yield "sdpa", lambda: pins.test_single_chunk_is_full_attention(100, 64)
    yield "sdpa_odd_d", lambda: pins.test_single_chunk_is_full_attention(102, 7)
    for s in range(2):
        yield f"later_invisible[{s}]", lambda s=s: pins.test_later_chunks_are_invisible_bitwise(s)
    yield "no_leak", pins.test_values_of_a_later_chunk_never_leak
    for s in range(3):
        yield f"prefix_mean[{s}]", lambda s=s: pins.test_zero_queries_give_prefix_mean(s)
    yield "one_hot", lambda: pins.test_softmax_rows_via_one_hot_values(0)


def failing_pins(lib):
    saved = oracle._lib
    oracle._lib = lib
    failed = []
    try:
        for name, fn in battery():
            try:
                fn()
            except AssertionError:
                failed.append(name)
    finally:
        oracle._lib = saved
    return failed


@pytest.fixture(scope="module")
def workdir():
    d = tempfile.mkdtemp(prefix="oracle_mutants_")
    yield d
    shutil.rmtree(d, ignore_errors=True)


def test_unmutated_copy_passes_every_pin(workdir):
    path = os.path.join(workdir, "liboracle_copy.so")
    oracle.build(SRC, path)
    assert failing_pins(oracle.load_library(path)) == []


@pytest.mark.parametrize("name,find,repl", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(workdir, name, find, repl):
    text = open(SRC).read()
    assert find in text, f"mutation site for {name} not found"
    src = os.path.join(workdir, f"{name}.c")
    with open(src, "w") as f:
        f.write(text.replace(find, repl))
    lib_path = os.path.join(workdir, f"lib{name}.so")
    oracle.build(src, lib_path)
    failed = failing_pins(oracle.load_library(lib_path))
    assert failed, f"mutant {name} passed every pin"


# ----------------------------------------------------------------- paged-layout mutants (NumPy)
def _bad_scatter_row(pool, page_table, token_start, rows):
    ps = pool.shape[1]
    for i in range(rows.shape[0]):
        t = token_start + i
        pool[int(page_table[t // ps]), (t + 1) % ps] = rows[i]


def _bad_scatter_page(pool, page_table, token_start, rows):
    ps = pool.shape[1]
    for i in range(rows.shape[0]):
        t = token_start + i
        pool[int(page_table[min(t // ps + 1, len(page_table) - 1)]), t % ps] = rows[i]


@pytest.mark.parametrize("bad", [_bad_scatter_row, _bad_scatter_page])
def test_paging_mutant_is_caught(bad, monkeypatch):
    monkeypatch.setattr(oracle, "scatter_chunk", bad)
    with pytest.raises(AssertionError):
        pins.test_paging_golden_case()
