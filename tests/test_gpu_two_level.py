"""Parity of the two-level combine of a deduplicated dispatch (partition-side
reduce, token-side sum) with the oracle: partition rows bit-exact, token
rows within one bf16 step (expected: identical)."""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import (POISON_BYTE, compare_layout, compare_two_level, poisoned_buffers, problem_of,
                         to_dev, two_level_all_tokens)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _run(w, idx, po, gates, x, y):
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.z = torch.empty((max(prob.capacity, 1), prob.N), dtype=torch.bfloat16, device=DEV)
    b.z.view(torch.uint8).fill_(POISON_BYTE)
    b.layout_(to_dev(idx), to_dev(po))
    b.combine_two_level_(y, to_dev(gates))
    torch.cuda.synchronize()
    R_disp = int(b.layout.part_offset[prob.E_part].item())
    assert bool((b.z[R_disp:].view(torch.uint8) == POISON_BYTE).all()), "z written past R_disp"
    return prob, b


def test_hotpairs_workload_full():
    w = W.get("M16384-hotpairs-dedup")
    d = W.make_inputs(w, device=DEV)
    prob, b = _run(w, d["topk_idx"], d["part_of"], d["topk_weights"], d["x"], d["y"])
    ref = oracle.layout(d["topk_idx"], d["part_of"], w.G, w.E_part, True)
    compare_layout(b, ref, prob)
    assert two_level_all_tokens(b, prob, d["y"], d["topk_weights"], d["topk_idx"], d["part_of"],
                                ref) == 0


def test_prefill_workload_full():
    """Every token of the prefill batch: all z rows bit-exact, every out row
    within one bf16 step (expected: identical)."""
    w = W.get("prefill-M65536-mix-dedup-fp8")
    d = W.make_inputs(w, device=DEV)
    prob, b = _run(w, d["topk_idx"], d["part_of"], d["topk_weights"], d["x"], d["y"])
    ref = oracle.layout(d["topk_idx"], d["part_of"], w.G, w.E_part, True)
    compare_layout(b, ref, prob)
    assert two_level_all_tokens(b, prob, d["y"], d["topk_weights"], d["topk_idx"], d["part_of"],
                                ref) == 0


@pytest.mark.parametrize("M,N,G,topk,E", [(1, 128, 4, 2, 2), (37, 136, 10, 3, 4), (1000, 256, 7, 7, 3),
                                          (257, 128, 64, 1, 64), (300, 512, 1024, 32, 64),
                                          (2000, 64, 16, 9, 4)])
def test_shapes(M, N, G, topk, E):
    w = W.Workload("two-level", M=M, N=N, G=G, topk=topk, E_part=E, routing="uniform",
                   placement="contiguous", dedup=True, seed=M + topk)
    d = W.make_inputs(w, device=DEV)
    po = np.random.default_rng(M).permutation(d["part_of"]).astype(np.int32)
    prob, b = _run(w, d["topk_idx"], po, d["topk_weights"], d["x"], d["y"])
    ref = oracle.layout(d["topk_idx"], po, G, E, True)
    assert compare_two_level(b, prob, d["y"], d["topk_weights"], d["topk_idx"], po, ref) == 0


def test_invalid_ids_are_left_out():
    w = W.Workload("two-level-bad", M=300, N=128, G=32, topk=4, E_part=4, routing="uniform",
                   placement="contiguous", dedup=True, seed=3)
    d = W.make_inputs(w, device=DEV)
    idx = d["topk_idx"].copy()
    idx[5, 2] = 99
    idx[17, 0] = -4
    prob, b = _run(w, idx, d["part_of"], d["topk_weights"], d["x"], d["y"])
    ref = oracle.layout(idx, d["part_of"], w.G, w.E_part, True)
    assert ref["status"] == moe.MOE_STATUS_BAD_EXPERT
    compare_layout(b, ref, prob)
    assert compare_two_level(b, prob, d["y"], d["topk_weights"], idx, d["part_of"], ref) == 0


def test_needs_a_dedup_layout():
    prob = moe.MoEProblem(64, 128, 8, 2, 2, dedup=False)
    b = moe.MoEBuffers(prob, DEV)
    y = torch.zeros((128, 128), dtype=torch.bfloat16, device=DEV)
    g = torch.zeros((64, 2), dtype=torch.float32, device=DEV)
    with pytest.raises(ValueError):
        moe.moe_combine_partial(prob, y, g, b.layout, y)
    import ctypes
    from combine_moe_layout_08_b200 import _lib
    s, l = prob.struct(), b.layout.struct()
    assert _lib.load().moe_combine_partial(ctypes.byref(s), y.data_ptr(), g.data_ptr(),
                                           ctypes.byref(l), y.data_ptr(), None) == 1
    assert _lib.load().moe_combine_reduce(ctypes.byref(s), y.data_ptr(), ctypes.byref(l),
                                          b.out.data_ptr(), None) == 1
