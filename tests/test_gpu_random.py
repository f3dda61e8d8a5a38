"""Seeded random problems through every entry point, against the oracle.

Forty small problems with sizes and options drawn from one seeded generator
(M, N, G, topk, E_part, dedup, fp8, routing, placement, the schedule, the
tile size), each run through layout + dispatch (one call or two), the
combine (one-level, and two-level with dedup) and the tile metadata, and
compared with the oracle: layout, rows, FP8 bytes and scales, partition rows
and tiles bit-exact, combine within one bf16 step (expected: identical).
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import (POISON_I32, compare_combine, compare_dispatch_rows, compare_layout,
                         compare_two_level, poisoned_buffers, problem_of, to_dev,
                         untouched_rows_ok)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(i):
    rng = np.random.default_rng(1000 + i)
    fp8 = bool(rng.random() < 0.4)
    N = int(rng.integers(1, 9)) * (128 if fp8 else 8 * int(rng.choice([1, 3, 16, 56])))
    G = int(rng.choice([1, 3, 8, 37, 128, 256, 1000]))
    topk = int(rng.integers(1, min(G, 32) + 1))
    E = int(rng.integers(1, 65))
    M = int(rng.choice([1, 7, 63, 129, 600, 1500, 3000]))
    return dict(M=M, N=N, G=G, topk=topk, E_part=E, dedup=bool(rng.random() < 0.5), fp8=fp8,
                routing=str(rng.choice(["uniform", "zipf", "mix"])),
                separate=bool(rng.random() < 0.3), block_m=int(rng.choice([1, 16, 128])),
                seed=int(rng.integers(0, 1 << 30)))


@pytest.mark.parametrize("i", range(40))
def test_random_problem(i):
    c = _case(i)
    w = W.Workload(f"random{i}", M=c["M"], N=c["N"], G=c["G"], topk=c["topk"], E_part=c["E_part"],
                   routing=c["routing"], placement="contiguous", dedup=c["dedup"], fp8=c["fp8"],
                   zipf_s=1.2, seed=c["seed"])
    d = W.make_inputs(w, device=DEV)
    po = np.random.default_rng(c["seed"]).integers(0, c["E_part"], size=c["G"]).astype(np.int32)
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.tiles = moe.alloc_expert_tiles(prob, c["block_m"], DEV)
    for t in (b.tiles.tile_first, b.tiles.tile_expert, b.tiles.tile_row, b.tiles.tile_rows):
        t.fill_(POISON_I32)
    idx, po_d, g = to_dev(d["topk_idx"]), to_dev(po), to_dev(d["topk_weights"])
    if c["separate"]:
        b.layout_(idx, po_d)
        b.dispatch_(d["x"])
        b.expert_tiles_(po_d, c["block_m"])
    else:
        b.layout_dispatch_(idx, po_d, d["x"], block_m=c["block_m"])
    b.combine_(d["y"], g)
    torch.cuda.synchronize()

    ref = oracle.layout(d["topk_idx"], po, w.G, w.E_part, w.dedup)
    compare_layout(b, ref, prob)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(d["x"]), ref["disp_token"])
    untouched_rows_ok(b, ref["R_disp"])
    assert compare_combine(b, prob, d["y"], d["topk_weights"], ref["exp_row"]) == 0
    tiles = oracle.expert_tiles(ref["expert_count"], ref["expert_offset"], c["block_m"])
    n = tiles["n_tiles"]
    np.testing.assert_array_equal(b.tiles.tile_first.cpu().numpy(), tiles["tile_first"])
    for name in ("tile_expert", "tile_row", "tile_rows"):
        got = getattr(b.tiles, name).cpu().numpy()
        np.testing.assert_array_equal(got[:n], tiles[name])
        assert np.all(got[n:] == POISON_I32)
    if c["dedup"]:
        b.z = torch.empty((max(prob.capacity, 1), prob.N), dtype=torch.bfloat16, device=DEV)
        b.combine_two_level_(d["y"], g)
        torch.cuda.synchronize()
        assert compare_two_level(b, prob, d["y"], d["topk_weights"], d["topk_idx"], po, ref) == 0


# duplicate expert ids inside a token (reading: separate rows, ranked by
# slot), through the one-kernel and the separate schedules, the two-level
# combine (duplicates fall in one partition group) and the tile metadata
@pytest.mark.parametrize("M,topk,separate", [(200, 8, False), (200, 8, True), (3000, 4, False)])
@pytest.mark.parametrize("pattern", ["one-expert", "few-experts", "one-partition"])
def test_duplicate_expert_ids(M, topk, separate, pattern):
    w = W.Workload("dups", M=M, N=256, G=16, topk=topk, E_part=8, routing="uniform",
                   placement="contiguous", dedup=True, fp8=(topk == 4), seed=M + topk)
    d = W.make_inputs(w, device=DEV)
    rng = np.random.default_rng(M * 3 + topk)
    po = W.make_placement(w)
    if pattern == "one-expert":
        idx = np.full((M, topk), 5, np.int32)
    elif pattern == "few-experts":
        idx = rng.integers(0, 3, size=(M, topk)).astype(np.int32)
    else:
        idx = rng.integers(0, 16, size=(M, topk)).astype(np.int32)
        po = np.zeros_like(po)
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.tiles = moe.alloc_expert_tiles(prob, 16, DEV)
    for t in (b.tiles.tile_first, b.tiles.tile_expert, b.tiles.tile_row, b.tiles.tile_rows):
        t.fill_(POISON_I32)
    idx_d, po_d, g = to_dev(idx), to_dev(po), to_dev(d["topk_weights"])
    if separate:
        b.layout_(idx_d, po_d)
        b.dispatch_(d["x"])
        b.expert_tiles_(po_d, 16)
    else:
        b.layout_dispatch_(idx_d, po_d, d["x"], block_m=16)
    b.combine_(d["y"], g)
    torch.cuda.synchronize()
    ref = oracle.layout(idx, po, w.G, w.E_part, True)
    compare_layout(b, ref, prob)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(d["x"]), ref["disp_token"])
    untouched_rows_ok(b, ref["R_disp"])
    assert compare_combine(b, prob, d["y"], d["topk_weights"], ref["exp_row"]) == 0
    tiles = oracle.expert_tiles(ref["expert_count"], ref["expert_offset"], 16)
    np.testing.assert_array_equal(b.tiles.tile_first.cpu().numpy(), tiles["tile_first"])
    np.testing.assert_array_equal(b.tiles.tile_expert.cpu().numpy()[:tiles["n_tiles"]],
                                  tiles["tile_expert"])
    b.z = torch.empty((max(prob.capacity, 1), prob.N), dtype=torch.bfloat16, device=DEV)
    b.combine_two_level_(d["y"], g)
    torch.cuda.synchronize()
    assert compare_two_level(b, prob, d["y"], d["topk_weights"], idx, po, ref) == 0
