"""moe_layout_static: the layout entry point that allocates nothing.

Some callers cannot allocate device memory where they route tokens -- code
inside a CUDA-graph capture that must not call cudaMalloc, runtimes whose
memory planner hands out no scratch, plain C hosts without an allocator.
For them the layout's scratch is a fixed device array inside the library.
This file checks, through the C ABI, that the entry point gives exactly the
layout moe_layout gives (with a caller workspace) on two calls in a row with
different inputs, and that a problem needing more scratch than the array
holds is refused before any launch.  It is collected last on purpose.
"""
import ctypes

import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import workloads as W
from combine_moe_layout_08_b200 import _lib

pytestmark = pytest.mark.gpu

FIELDS = ("expert_count", "expert_offset", "part_count", "part_offset", "exp_row",
          "disp_token", "disp_row", "exp_to_disp", "status")


def _static(prob, idx, po, lay, stream):
    s, l = prob.struct(), lay.struct()
    return _lib.load().moe_layout_static(ctypes.byref(s), idx.data_ptr(), po.data_ptr(),
                                         ctypes.byref(l), stream)


def _with_workspace(prob, idx, po, lay, ws, stream):
    s, l = prob.struct(), lay.struct()
    return _lib.load().moe_layout(ctypes.byref(s), idx.data_ptr(), po.data_ptr(), ctypes.byref(l),
                                  ws.data_ptr(), ws.numel(), stream)


def _poisoned_layout(prob):
    lay = moe.alloc_layout(prob, "cuda")
    for f in FIELDS:
        t = getattr(lay, f)
        if t is not None:
            t.fill_(-7)
    return lay


@pytest.mark.parametrize("name", ["M4096-zipf1.1", "M16384-hotpairs-dedup",
                                  "prefill-M65536-mix-dedup-fp8"])
def test_static_scratch_layout_matches_workspace_layout(name):
    w = W.get(name)
    prob = moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)
    assert moe.layout_workspace_size(prob) <= moe.MOE_STATIC_SCRATCH_BYTES
    stream = torch.cuda.current_stream().cuda_stream
    ws = torch.empty(moe.layout_workspace_size(prob), dtype=torch.uint8, device="cuda")
    for call in range(2):                       # two calls in a row, different inputs
        wc = w.replace(seed=call)
        idx = torch.from_numpy(W.make_routing(wc)).cuda()
        po = torch.from_numpy(W.make_placement(wc)).cuda()
        want, got = _poisoned_layout(prob), _poisoned_layout(prob)
        assert _with_workspace(prob, idx, po, want, ws, stream) == 0
        assert _static(prob, idx, po, got, stream) == 0
        torch.cuda.synchronize()
        for f in FIELDS:
            a, b = getattr(want, f), getattr(got, f)
            if a is not None:
                assert torch.equal(a, b), f"call {call}: {f} differs"
        assert got.status.item() == 0


def test_static_scratch_refuses_problem_beyond_its_size():
    prob = moe.MoEProblem(65536, 7168, 1024, 8, 64, dedup=True)
    assert moe.layout_workspace_size(prob) > moe.MOE_STATIC_SCRATCH_BYTES
    lay = _poisoned_layout(prob)
    idx = torch.zeros((prob.M, prob.topk), dtype=torch.int32, device="cuda")
    po = torch.zeros(prob.G, dtype=torch.int32, device="cuda")
    rc = _static(prob, idx, po, lay, torch.cuda.current_stream().cuda_stream)
    assert rc == 2                               # MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert int(lay.status.item()) == -7          # nothing was launched
    assert np.all(lay.exp_row[:16].cpu().numpy() == -7)
