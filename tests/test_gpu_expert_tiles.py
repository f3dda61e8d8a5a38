"""Parity of moe_expert_tiles (grouped-GEMM tile metadata of a layout) with
the oracle, through the C ABI: tile_first and every tile's expert, first row
and rows bit-exact, entries past the number of tiles untouched, and counts
that no layout of the problem gives written only up to capacity and flagged."""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import POISON_I32, poisoned_buffers, problem_of, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _tiles(prob, block_m, guard=0):
    cap = moe.expert_tiles_capacity(prob, block_m)
    i32 = dict(dtype=torch.int32, device=DEV)
    t = moe.ExpertTiles(block_m, torch.full((prob.G + 1,), POISON_I32, **i32),
                        *(torch.full((cap + guard,), POISON_I32, **i32) for _ in range(3)))
    return t, cap


def _compare(t, ref):
    n = ref["n_tiles"]
    np.testing.assert_array_equal(t.tile_first.cpu().numpy(), ref["tile_first"])
    for name in ("tile_expert", "tile_row", "tile_rows"):
        got = getattr(t, name).cpu().numpy()
        np.testing.assert_array_equal(got[:n], ref[name], err_msg=name)
        assert np.all(got[n:] == POISON_I32), f"{name} written past the last tile"


@pytest.mark.parametrize("name", ["decode-M128-uniform", "M4096-zipf1.1", "M16384-hotpairs-dedup",
                                  "prefill-M65536-mix-dedup-fp8"])
@pytest.mark.parametrize("block_m", [1, 64, 128, 256])
def test_workloads(name, block_m):
    w = W.get(name)
    prob = problem_of(w)
    idx, po = W.make_routing(w), W.make_placement(w)
    b = poisoned_buffers(prob, DEV)
    b.layout_(to_dev(idx), to_dev(po))
    t, _ = _tiles(prob, block_m)
    moe.moe_expert_tiles(prob, to_dev(po), b.layout, t)
    torch.cuda.synchronize()
    lay = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    _compare(t, oracle.expert_tiles(lay["expert_count"], lay["expert_offset"], block_m))
    assert int(b.layout.status.item()) == 0


@pytest.mark.parametrize("block_m", [1, 5, 128])
def test_unplaced_and_empty_experts(block_m):
    w = W.Workload("tiles-odd", M=333, N=64, G=1024, topk=3, E_part=64, routing="zipf",
                   placement="contiguous", zipf_s=1.3, seed=9)
    prob = problem_of(w)
    idx = W.make_routing(w)
    po = np.random.default_rng(4).permutation(W.make_placement(w)).astype(np.int32)
    po[[0, 17, 999]] = 64                            # placed nowhere
    b = poisoned_buffers(prob, DEV)
    b.layout_(to_dev(idx), to_dev(po))
    t, _ = _tiles(prob, block_m)
    moe.moe_expert_tiles(prob, to_dev(po), b.layout, t)
    torch.cuda.synchronize()
    lay = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    _compare(t, oracle.expert_tiles(lay["expert_count"], lay["expert_offset"], block_m))


def test_counts_beyond_capacity_are_bounded_and_flagged():
    w = W.Workload("tiles-bad", M=64, N=64, G=32, topk=2, E_part=4, routing="uniform",
                   placement="contiguous", seed=2)
    prob = problem_of(w)
    idx, po = W.make_routing(w), W.make_placement(w)
    b = poisoned_buffers(prob, DEV)
    b.layout_(to_dev(idx), to_dev(po))
    b.layout.expert_count.fill_(prob.M * prob.topk)   # no layout of this problem has these
    t, cap = _tiles(prob, 4, guard=64)
    moe.moe_expert_tiles(prob, to_dev(po), b.layout, t)
    torch.cuda.synchronize()
    assert int(b.layout.status.item()) & moe.MOE_STATUS_BAD_ROW
    for name in ("tile_expert", "tile_row", "tile_rows"):
        got = getattr(t, name).cpu().numpy()
        assert np.all(got[cap:] == POISON_I32) and np.all(got[:cap] != POISON_I32)


def test_empty_batch():
    prob = moe.MoEProblem(0, 64, 16, 2, 4)
    b = poisoned_buffers(prob, DEV)
    po = torch.arange(16, dtype=torch.int32, device=DEV) % 4
    b.layout_(torch.zeros(1, dtype=torch.int32, device=DEV), po)
    t, _ = _tiles(prob, 128)
    moe.moe_expert_tiles(prob, po, b.layout, t)
    torch.cuda.synchronize()
    assert np.all(t.tile_first.cpu().numpy() == 0)
    assert np.all(t.tile_expert.cpu().numpy() == POISON_I32)


# tiles emitted by moe_layout_dispatch from inside each layout schedule
@pytest.mark.parametrize("M,G,topk,E,dedup,fp8", [
    (128, 256, 8, 8, False, False),    # one kernel for layout + dispatch
    (900, 256, 8, 8, True, False),     # one-cluster layout (7200 pairs)
    (4096, 256, 8, 8, False, True),    # two-launch tiled layout
    (3000, 1024, 32, 64, True, False),  # largest G / topk / E_part, tiled
])
@pytest.mark.parametrize("block_m", [1, 128])
def test_tiles_from_layout_dispatch(M, G, topk, E, dedup, fp8, block_m):
    from gpu_harness import compare_dispatch_rows, compare_layout, untouched_rows_ok
    w = W.Workload("tiles-ld", M=M, N=128, G=G, topk=topk, E_part=E, routing="zipf",
                   placement="contiguous", dedup=dedup, fp8=fp8, zipf_s=1.2, seed=M + block_m)
    prob = problem_of(w)
    d = W.make_inputs(w, device=DEV, with_y=False)
    po = np.random.default_rng(M).permutation(d["part_of"]).astype(np.int32)
    b = poisoned_buffers(prob, DEV)
    t, _ = _tiles(prob, block_m)
    b.tiles = t
    b.layout_dispatch_(to_dev(d["topk_idx"]), to_dev(po), d["x"], block_m=block_m)
    torch.cuda.synchronize()
    lay = oracle.layout(d["topk_idx"], po, G, E, dedup)
    compare_layout(b, lay, prob)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(d["x"]), lay["disp_token"])
    untouched_rows_ok(b, lay["R_disp"])
    _compare(t, oracle.expert_tiles(lay["expert_count"], lay["expert_offset"], block_m))
