"""Parity of moe_layout_dispatch (layout and dispatch in one call; one kernel
for small batches) with the oracle, through the C ABI: layout arrays,
dispatched rows, FP8 bytes and scales bit-exact, rows past R_disp untouched.
Covers the decode batch, the boundaries of the one-kernel schedule, chunks
of several tokens per block, rows split across blocks, dedup and FP8, the
largest G / topk / E_part, invalid input and graph capture."""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import (POISON_I32, compare_dispatch_rows, compare_layout, poisoned_buffers,
                         problem_of, to_dev, untouched_rows_ok)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(w, idx, po, x):
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.layout_dispatch_(to_dev(idx), to_dev(po), x)
    torch.cuda.synchronize()
    return prob, b


def _check(w, idx, po, x):
    prob, b = _run(w, idx, po, x)
    ref = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    compare_layout(b, ref, prob)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(x), ref["disp_token"])
    untouched_rows_ok(b, ref["R_disp"])
    return prob, b, ref


def test_decode_workload_is_one_kernel_and_exact():
    w = W.get("decode-M128-uniform")
    d = W.make_inputs(w, device=DEV)
    assert moe.moe_layout_dispatch_fused(problem_of(w))
    _check(w, d["topk_idx"], d["part_of"], d["x"])


# (M, N, G, topk, E, dedup, fp8, routing)
SHAPES = [
    (1, 128, 4, 2, 2, False, False, "uniform"),
    (1, 256, 8, 8, 8, True, True, "uniform"),
    (2, 7168, 256, 8, 8, False, False, "uniform"),     # the smallest batch of the pages' table
    (149, 256, 64, 4, 8, True, False, "zipf"),         # two tokens per block, ragged last chunk
    (300, 1024, 256, 8, 8, False, True, "zipf"),       # three tokens per block, fp8
    (512, 7168, 256, 8, 8, True, True, "mix"),         # 4096 pairs: largest one-kernel batch
    (513, 7168, 256, 8, 8, False, False, "uniform"),   # 4104 pairs: separate kernels
    (2048, 64, 16, 2, 4, True, False, "uniform"),      # 14 tokens per block
    (4096, 64, 128, 1, 8, False, False, "zipf"),       # 16 tokens per block (the cap)
    (100, 65536, 32, 3, 4, False, False, "uniform"),   # each chunk split over two blocks
    (64, 32768, 128, 5, 8, True, True, "zipf"),        # fp8, 2048 units per row
    (128, 128, 1024, 32, 64, True, False, "uniform"),  # largest G, topk, E_part
    (90, 136, 10, 3, 4, True, False, "uniform"),       # N not a multiple of 128
]


@pytest.mark.parametrize("M,N,G,topk,E,dedup,fp8,routing", SHAPES)
def test_shapes(M, N, G, topk, E, dedup, fp8, routing):
    w = W.Workload(f"ld{M}", M=M, N=N, G=G, topk=topk, E_part=E, routing=routing,
                   placement="contiguous", dedup=dedup, fp8=fp8, zipf_s=1.1, seed=3 * M + N)
    d = W.make_inputs(w, device=DEV, with_y=False)
    po = np.random.default_rng(M + 1).permutation(d["part_of"]).astype(np.int32)
    prob = problem_of(w)
    assert moe.moe_layout_dispatch_fused(prob) == (M * topk <= 4096)
    _check(w, d["topk_idx"], po, d["x"])


def test_same_bits_as_separate_calls():
    w = W.Workload("ld-vs-separate", M=200, N=1024, G=64, topk=6, E_part=8, routing="zipf",
                   placement="contiguous", dedup=True, fp8=True, zipf_s=1.2, seed=11)
    d = W.make_inputs(w, device=DEV, with_y=False)
    prob = problem_of(w)
    idx, po = to_dev(d["topk_idx"]), to_dev(d["part_of"])
    a = poisoned_buffers(prob, DEV)
    a.layout_dispatch_(idx, po, d["x"])
    b = poisoned_buffers(prob, DEV)
    b.layout_(idx, po)
    b.dispatch_(d["x"])
    torch.cuda.synchronize()
    for name in ("expert_count", "expert_offset", "part_count", "part_offset", "exp_row",
                 "disp_token", "status", "disp_row", "exp_to_disp"):
        assert torch.equal(getattr(a.layout, name), getattr(b.layout, name)), name
    assert torch.equal(a.recv_x, b.recv_x)
    assert torch.equal(a.recv_scale.view(torch.int32), b.recv_scale.view(torch.int32))


@pytest.mark.parametrize("dedup", [False, True])
def test_invalid_input_is_left_out_and_flagged(dedup):
    w = W.Workload("ld-bad", M=96, N=256, G=32, topk=4, E_part=4, routing="uniform",
                   placement="contiguous", dedup=dedup, seed=5)
    d = W.make_inputs(w, device=DEV, with_y=False)
    idx = d["topk_idx"].copy()
    idx[3, 1] = 32
    idx[50, 0] = -9
    po = d["part_of"].copy()
    po[7] = 4                                    # expert 7 placed nowhere
    prob, b, ref = _check(w, idx, po, d["x"])
    assert ref["status"] == moe.MOE_STATUS_BAD_EXPERT | moe.MOE_STATUS_BAD_PART
    assert int(b.layout.status.item()) == ref["status"]


def test_repeat_and_graph_capture():
    w = W.get("decode-M128-uniform")
    d = W.make_inputs(w, device=DEV, with_y=False)
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    idx, po = to_dev(d["topk_idx"]), to_dev(d["part_of"])
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b.layout_dispatch_(idx, po, d["x"])
    s.synchronize()
    first = b.recv_x.clone(), b.layout.exp_row.clone()
    b.recv_x.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.layout_dispatch_(idx, po, d["x"])
    for _ in range(3):
        g.replay()
    torch.cuda.synchronize()
    assert torch.equal(b.recv_x, first[0]) and torch.equal(b.layout.exp_row, first[1])


@pytest.mark.parametrize("dedup,fp8", [(False, False), (True, True)])
def test_empty_batch(dedup, fp8):
    """M = 0: counts and offsets all zero, status 0, no row written, no tiles."""
    prob = moe.MoEProblem(0, 256, 16, 4, 4, dedup, fp8)
    assert not moe.moe_layout_dispatch_fused(prob)
    b = poisoned_buffers(prob, DEV)
    b.tiles = moe.alloc_expert_tiles(prob, 64, DEV)
    for t in (b.tiles.tile_first, b.tiles.tile_expert, b.tiles.tile_row, b.tiles.tile_rows):
        t.fill_(POISON_I32)
    po = torch.arange(16, dtype=torch.int32, device=DEV) % 4
    x = torch.zeros((1, 256), dtype=torch.bfloat16, device=DEV)
    b.layout_dispatch_(torch.zeros(1, dtype=torch.int32, device=DEV), po, x, block_m=64)
    torch.cuda.synchronize()
    assert int(b.layout.status.item()) == 0
    for t in (b.layout.expert_count, b.layout.expert_offset, b.layout.part_count,
              b.layout.part_offset, b.tiles.tile_first):
        assert bool((t == 0).all())
    assert bool((b.tiles.tile_expert == POISON_I32).all())


def test_binding_rejects_bad_tensors():
    w = W.get("decode-M128-uniform")
    prob = problem_of(w)
    d = W.make_inputs(w, device=DEV, with_y=False)
    b = moe.MoEBuffers(prob, DEV)
    idx, po = to_dev(d["topk_idx"]), to_dev(d["part_of"])
    with pytest.raises(TypeError):
        b.layout_dispatch_(idx.long(), po, d["x"])
    with pytest.raises(ValueError):
        b.layout_dispatch_(idx, po, d["x"][:, ::2])            # not contiguous
    with pytest.raises(ValueError):
        b.layout_dispatch_(idx, po, d["x"][:64])               # too few rows
    with pytest.raises(ValueError):
        moe.alloc_expert_tiles(prob, 0, DEV)                   # block_m < 1
    t = moe.alloc_expert_tiles(prob, 128, DEV)
    t.tile_row = t.tile_row[:10]
    with pytest.raises(ValueError):
        moe.moe_layout_dispatch(prob, idx, po, b.layout, b.workspace, d["x"], b.recv_x, tiles=t)


def test_replaced_buffers_are_checked_again():
    """MoEBuffers checks its own buffers once, and again after one is replaced."""
    w = W.get("decode-M128-uniform")
    prob = problem_of(w)
    d = W.make_inputs(w, device=DEV)
    idx, po, g = to_dev(d["topk_idx"]), to_dev(d["part_of"]), to_dev(d["topk_weights"])
    b = moe.MoEBuffers(prob, DEV)
    b.layout_dispatch_(idx, po, d["x"])
    b.recv_x = b.recv_x[:10]                                   # too few rows
    with pytest.raises(ValueError):
        b.layout_dispatch_(idx, po, d["x"])
    b = moe.MoEBuffers(prob, DEV)
    b.layout_dispatch_(idx, po, d["x"])
    b.layout.exp_row = b.layout.exp_row[:5]                    # too short
    with pytest.raises(ValueError):
        b.combine_(d["y"], g)
    b = moe.MoEBuffers(prob, DEV)
    b.out = b.out.float()                                      # wrong dtype
    with pytest.raises(TypeError):
        b.step(idx, po, d["x"], d["y"], g)


@pytest.mark.parametrize("M,topk,dedup", [(128, 8, False),     # one kernel
                                          (1000, 8, True),     # one-cluster layout
                                          (4096, 8, False)])   # two-launch tiled layout
def test_routing_ids_not_16_byte_aligned(M, topk, dedup):
    """topk_idx starting 4 bytes past a 16-byte boundary takes the scalar
    staging path of every layout schedule; the results are the same."""
    w = W.Workload("ld-unaligned", M=M, N=64, G=256, topk=topk, E_part=8, routing="zipf",
                   placement="contiguous", dedup=dedup, zipf_s=1.1, seed=M)
    d = W.make_inputs(w, device=DEV, with_y=False)
    flat = torch.empty(M * topk + 1, dtype=torch.int32, device=DEV)
    idx = flat[1:].view(M, topk)
    idx.copy_(to_dev(d["topk_idx"]))
    assert idx.data_ptr() % 16 == 4
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.layout_dispatch_(idx, to_dev(d["part_of"]), d["x"])
    torch.cuda.synchronize()
    ref = oracle.layout(d["topk_idx"], d["part_of"], w.G, w.E_part, w.dedup)
    compare_layout(b, ref, prob)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(d["x"]), ref["disp_token"])
