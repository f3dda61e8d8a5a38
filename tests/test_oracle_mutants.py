"""The pins must catch plausible mistakes in the oracle.

Each mutant is a textual edit of a temporary copy of ``oracle/moe_oracle.c``
(a swapped comparison, an off-by-one, a dropped term, a wrong sign, index or
constant), compiled with the oracle's own flags and swapped in for the real
library while the pin checks run.  Every mutant must fail at least one pin;
the committed oracle is never modified.
"""
import ctypes
import os
import subprocess

import numpy as np
import pytest

import oracle
from oracle import build as obuild

import test_oracle_combine as C
import test_oracle_ep as EP
import test_oracle_fp8 as F
import test_golden as GD
import test_oracle_layout as L
import test_oracle_tiles as T

SRC = open(obuild.SRC).read()

# (name, anchor to search from, old text, new text)
MUTANTS = [
    ("tie-break t reversed", "orc_cmp_pair", "return x->t < y->t ? -1 : 1;", "return x->t > y->t ? -1 : 1;"),
    ("expert key dropped", "orc_cmp_pair", "if (x->e != y->e) return x->e < y->e ? -1 : 1;", ""),
    ("k order reversed", "orc_cmp_pair", "return x->k < y->k ? -1 : 1;", "return x->k > y->k ? -1 : 1;"),
    ("inclusive expert offsets", "run = 0;",
     "expert_offset[e] = (int32_t)run;\n            run += expert_count[e];",
     "run += expert_count[e];\n            expert_offset[e] = (int32_t)run;"),
    ("dedup row off by one", "distinct (t, p)", "disp_row[j] = (int32_t)d;", "disp_row[j] = (int32_t)d + 1;"),
    ("dedup keyed by expert", "distinct (t, p)",
     "has[(int64_t)pairs[r].t * E_part + pairs[r].p] = 1;",
     "has[(int64_t)pairs[r].t * E_part + (pairs[r].e % E_part)] = 1;"),
    ("e4m3 ties away", "orc_round_half_even(float q)", "else if (frac == 0.5f) n += (n & 1);",
     "else if (frac == 0.5f) n += 1;"),
    ("e4m3 subnormal quantum", "below 2^-6", "a * 512.0f", "a * 256.0f"),
    ("e4m3 no saturation", "static uint8_t orc_e4m3", "if (E > 8 || code > 0x7E) code = 0x7E;", ""),
    ("scale constant", "orc_quantize_block", "amax / 448.0f", "amax / 240.0f"),
    ("bf16 ties away", "orc_f32_to_bf16(float f)", "u += 0x7FFFu + lsb;", "u += 0x8000u;"),
    ("combine drops last k", "int oracle_combine", "for (int32_t k = 0; k < topk; ++k)",
     "for (int32_t k = 0; k < topk - 1; ++k)"),
    ("combine gate index", "int oracle_combine", "float wk = w[t * topk + k];",
     "float wk = w[t * topk + (topk - 1 - k)];"),
    ("combine gate sign", "int oracle_combine", "acc[c] = fmaf(wk,", "acc[c] = fmaf(-wk,"),
    ("combine token row", "int oracle_combine", "y + (int64_t)r * N", "y + (int64_t)t * N"),
    ("dispatch wrong row", "void oracle_dispatch", "x + (int64_t)disp_token[r] * N", "x + (int64_t)r * N"),
    ("partial: wrong partition test", "int oracle_combine_partial", "part_of[e] != p", "part_of[e] == p"),
    ("partial: drops last slot", "int oracle_combine_partial", "for (int32_t k = 0; k < topk; ++k)",
     "for (int32_t k = 0; k < topk - 1; ++k)"),
    ("partial: gate sign", "int oracle_combine_partial", "acc[c] = fmaf(wk,", "acc[c] = fmaf(-wk,"),
    ("reduce: drops first partition", "int oracle_combine_reduce", "for (int32_t p = 0; p < E_part; ++p)",
     "for (int32_t p = 1; p < E_part; ++p)"),
    ("reduce: wrong row", "int oracle_combine_reduce", "z + (int64_t)r * N", "z + (int64_t)t * N"),
    ("tiles: ties before", "int64_t oracle_expert_tiles", "if (expert_offset[f] < expert_offset[e])",
     "if (expert_offset[f] <= expert_offset[e] && f != e)"),
    ("tiles: floor count", "int64_t n = ((int64_t)expert_count[e] + block_m - 1) / block_m;",
     "int64_t n = ((int64_t)expert_count[e] + block_m - 1) / block_m;",
     "int64_t n = (int64_t)expert_count[e] / block_m;"),
    ("tiles: full last tile", "int64_t oracle_expert_tiles", "(rest < block_m ? rest : block_m)", "(block_m)"),
    ("tiles: row start", "int64_t oracle_expert_tiles", "(expert_offset[e] + j * block_m)",
     "(expert_offset[e] + j * block_m + (j > 0))"),
    ("ep: send offset counts own rank", "void oracle_ep_plan", "for (int32_t s = 0; s < r; ++s)",
     "for (int32_t s = 0; s <= r; ++s)"),
    ("ep: source offset transposed", "void oracle_ep_plan",
     "for (int32_t d = 0; d < r; ++d) sum += part_counts[(int64_t)s * W + d];",
     "for (int32_t d = 0; d < r; ++d) sum += part_counts[(int64_t)d * W + s];"),
    ("ep: receive offsets transposed", "void oracle_ep_plan",
     "for (int32_t q = 0; q < s; ++q) sum += part_counts[(int64_t)q * W + r];",
     "for (int32_t q = 0; q < s; ++q) sum += part_counts[(int64_t)r * W + q];"),
    ("ep: receive count row", "void oracle_ep_plan", "recv_count[s] = part_counts[(int64_t)s * W + r];",
     "recv_count[s] = part_counts[(int64_t)r * W + s];"),
    ("ep: block counts its own expert", "void oracle_ep_plan", "for (int32_t f = 0; f < e; ++f)",
     "for (int32_t f = 0; f <= e; ++f)"),
]


def _mutate(anchor, old, new):
    i = SRC.index(anchor)
    j = SRC.index(old, i)
    return SRC[:j] + new + SRC[j + len(old):]


def _pins():
    """A quick cross-section of the oracle's pins."""
    return [
        lambda: L.test_layout_exhaustive_tiny(2, 2, 3, 2, (), False),
        lambda: L.test_layout_exhaustive_tiny(2, 2, 3, 2, (), True),
        lambda: L.test_layout_exhaustive_tiny(1, 3, 4, 2, (), False),
        lambda: L.test_layout_invariants(37, 3, 10, 4, True),
        lambda: F.test_e4m3_exhaustive_vs_table(1.0),
        lambda: F.test_e4m3_exhaustive_vs_table(2.0 ** 20),
        F.test_e4m3_saturation_and_signs,
        F.test_bf16_round_vs_torch,
        F.test_fp8_dispatch_scales_and_roundtrip,
        F.test_bf16_dispatch_identity,
        lambda: C.test_combine_one_hot_identity(3),
        lambda: C.test_combine_uniform_gates_identity(4),
        lambda: C.test_combine_within_fp64_bound(5),
        lambda: C.test_two_level_one_hot_identity(4),
        lambda: C.test_two_level_colocated_uniform_identity(4),
        lambda: C.test_two_level_within_fp64_bounds(5, 3),
        lambda: T.test_tiles_match_the_row_walk(1, 8, 2, 1, False, "random", 3),
        lambda: T.test_tiles_match_the_row_walk(200, 40, 8, 5, True, "random", 16),
        T.test_block_of_one_row_labels_every_row,
        GD.test_zyphra_hot_pairs_closed_forms,
        lambda: EP.test_exchange_by_definition_push_and_pull(3, 2, 12, 2, False),
        lambda: EP.test_exchange_by_definition_push_and_pull(4, 3, 16, 4, True),
        lambda: EP.test_expert_blocks_hold_each_sources_expert_rows(4, 3, 16, 4),
        EP.test_closed_forms,
    ]


def _load(src, tmp_path, tag):
    c = tmp_path / f"mut_{tag}.c"
    so = tmp_path / f"mut_{tag}.so"
    c.write_text(src)
    cmd = ["gcc", *obuild.CFLAGS, str(c), "-o", str(so), "-lm"]
    subprocess.run(cmd, check=True, capture_output=True)
    return str(so)


def _swap(path):
    """Point the oracle module at another build of the same source."""
    saved = oracle._lib
    oracle._lib = None
    real = obuild.build
    obuild.build = lambda *a, **k: path
    try:
        oracle.lib()
    finally:
        obuild.build = real
    return saved


@pytest.mark.parametrize("name,anchor,old,new", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(name, anchor, old, new, tmp_path):
    src = _mutate(anchor, old, new)
    assert src != SRC
    path = _load(src, tmp_path, abs(hash(name)) % 10 ** 8)
    saved = _swap(path)
    try:
        caught = 0
        for pin in _pins():
            try:
                pin()
            except AssertionError:
                caught += 1
                break
        assert caught, f"no pin caught mutant {name!r}"
    finally:
        oracle._lib = saved


def test_unmutated_copy_passes(tmp_path):
    path = _load(SRC, tmp_path, "same")
    saved = _swap(path)
    try:
        for pin in _pins():
            pin()
    finally:
        oracle._lib = saved
