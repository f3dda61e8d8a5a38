"""Layout code paths that the named workloads do not reach, against the oracle.

With dedup, a tile's (token, partition) rows are kept in shared memory for
the inverse map when ntok * E_part fits the free part of the reduction
buffer, and with E_part = 8 a token's eight rows are written as two 16-byte
stores when disp_row is 16-byte aligned.  These tests take the other sides:
  * tiles of 544 tokens x 8 partitions (M = 80,000): the rows no longer fit
    and the inverse map reads them back from global memory;
  * a disp_row that starts 4 bytes past a 16-byte boundary (E_part = 8): the
    rows go out one 4-byte store each, in the one-cluster schedule (M = 500)
    and in the tiled one (M = 4,096).
Every layout array is compared whole, bit-exact.
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import POISON_I32, compare_layout, poisoned_buffers, problem_of, to_dev

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _workload(M):
    # the prefill recipe's routing (half uniform, half Zipf) at M tokens,
    # rows of 8 columns (layout only)
    return W.Workload(f"paths-M{M}", M=M, N=8, G=256, topk=8, E_part=8, routing="mix",
                      placement="contiguous", dedup=True, fp8=False, zipf_s=1.2, seed=7)


def _oracle(w, d):
    return oracle.layout(d["topk_idx"], d["part_of"], w.G, w.E_part, w.dedup)


def test_dedup_rows_past_the_shared_copy():
    w = _workload(80_000)
    d = W.make_inputs(w, with_y=False)
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    b.layout_(to_dev(d["topk_idx"]), to_dev(d["part_of"]))
    torch.cuda.synchronize()
    compare_layout(b, _oracle(w, d), prob)


@pytest.mark.parametrize("M", [500, 4096])
def test_unaligned_disp_row(M):
    w = _workload(M)
    d = W.make_inputs(w, with_y=False)
    prob = problem_of(w)
    b = poisoned_buffers(prob, DEV)
    n = M * w.E_part
    raw = torch.full((n + 4,), POISON_I32, dtype=torch.int32, device=DEV)
    b.layout.disp_row = raw[1:1 + n]                 # 4 bytes past the allocation's start
    assert b.layout.disp_row.data_ptr() % 16 == 4
    b.layout_(to_dev(d["topk_idx"]), to_dev(d["part_of"]))
    torch.cuda.synchronize()
    compare_layout(b, _oracle(w, d), prob)
    assert int(raw[0].item()) == POISON_I32 and bool((raw[1 + n:] == POISON_I32).all())
