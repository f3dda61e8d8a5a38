"""moe_layout_static: the layout entry point that allocates nothing.

Some callers cannot allocate device memory where they route tokens -- code
inside a CUDA-graph capture that must not call cudaMalloc, runtimes whose
memory planner hands out no scratch, plain C hosts without an allocator.
For them the layout's scratch is a fixed device array inside the library.
This file checks, through the C ABI, that the entry point gives exactly the
layout moe_layout gives (with a caller workspace) on two calls in a row with
different inputs -- on the one-cluster schedule of a decode batch, which
leaves the scratch alone, and on the two-launch schedule, which uses it --
that a problem needing more scratch than the array holds is refused before
any launch, and that a plain C host which destroys and re-creates its CUDA
context between calls gets the same layout after the reset (the array's
address is looked up again in the new context).  It is collected last on
purpose.
"""
import ctypes
import os
import subprocess

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


@pytest.mark.parametrize("name", ["decode-M128-uniform", "M4096-zipf1.1",
                                  "M16384-hotpairs-dedup", "prefill-M65536-mix-dedup-fp8"])
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


C_RESET_HOST = r"""
#include <stdio.h>
#include <stdlib.h>
#include <string.h>
#include <cuda_runtime.h>
#include "moe_layout.h"

#define CK(x) do { if ((x) != cudaSuccess) { fprintf(stderr, "CUDA error at line %d\n", __LINE__); return 10; } } while (0)

enum { M = 4096, G = 256, K = 8, E = 8, NARR = 9 };

/* one layout with a workspace and one with the library's scratch, compared */
static int one_round(unsigned seed) {
    const size_t n = (size_t)M * K;
    const size_t sizes[NARR] = {G, G + 1, E, E + 1, n, n, (size_t)M * E, n, 1};
    moe_problem_t p = {M, 7168, G, K, E, 1, 0};
    int *h_idx = (int *)malloc(n * 4), *h_po = (int *)malloc(G * 4), *h_a = 0, *h_b = 0;
    int *d_idx = 0, *d_po = 0, *arr[2][NARR];
    void *ws = 0;
    size_t wsb = moe_layout_workspace_size(&p), i;
    int t, k, q, rc, a;
    unsigned s = seed * 2654435761u + 12345u;
    for (t = 0; t < M; ++t)            /* K distinct experts per token */
        for (k = 0; k < K; ++k) {
            int e, dup;
            do {
                s = s * 1664525u + 1013904223u;
                e = (int)((s >> 8) % G);
                for (dup = 0, q = 0; q < k; ++q) dup |= h_idx[t * K + q] == e;
            } while (dup);
            h_idx[t * K + k] = e;
        }
    for (i = 0; i < G; ++i) h_po[i] = (int)((i * 7 + seed) % E);
    CK(cudaMalloc((void **)&d_idx, n * 4));
    CK(cudaMalloc((void **)&d_po, G * 4));
    CK(cudaMalloc(&ws, wsb));
    CK(cudaMemcpy(d_idx, h_idx, n * 4, cudaMemcpyHostToDevice));
    CK(cudaMemcpy(d_po, h_po, G * 4, cudaMemcpyHostToDevice));
    for (a = 0; a < 2; ++a)
        for (i = 0; i < NARR; ++i) {
            CK(cudaMalloc((void **)&arr[a][i], sizes[i] * 4));
            CK(cudaMemset(arr[a][i], 0xA5, sizes[i] * 4));
        }
    {
        moe_layout_t l0 = {arr[0][0], arr[0][1], arr[0][2], arr[0][3], arr[0][4], arr[0][5],
                           arr[0][6], arr[0][7], arr[0][8]};
        moe_layout_t l1 = {arr[1][0], arr[1][1], arr[1][2], arr[1][3], arr[1][4], arr[1][5],
                           arr[1][6], arr[1][7], arr[1][8]};
        if ((rc = moe_layout(&p, d_idx, d_po, &l0, ws, wsb, 0)) != MOE_OK) return 20 + rc;
        if ((rc = moe_layout_static(&p, d_idx, d_po, &l1, 0)) != MOE_OK) return 30 + rc;
    }
    CK(cudaDeviceSynchronize());
    for (i = 0; i < NARR; ++i) {
        h_a = (int *)malloc(sizes[i] * 4);
        h_b = (int *)malloc(sizes[i] * 4);
        CK(cudaMemcpy(h_a, arr[0][i], sizes[i] * 4, cudaMemcpyDeviceToHost));
        CK(cudaMemcpy(h_b, arr[1][i], sizes[i] * 4, cudaMemcpyDeviceToHost));
        if (memcmp(h_a, h_b, sizes[i] * 4) != 0) {
            fprintf(stderr, "array %d differs in round %u\n", (int)i, seed);
            return 40;
        }
        if (i == 8 && h_a[0] != 0) return 41;   /* status */
        free(h_a);
        free(h_b);
    }
    for (a = 0; a < 2; ++a)
        for (i = 0; i < NARR; ++i) CK(cudaFree(arr[a][i]));
    CK(cudaFree(d_idx));
    CK(cudaFree(d_po));
    CK(cudaFree(ws));
    free(h_idx);
    free(h_po);
    return 0;
}

int main(void) {
    unsigned r;
    int rc;
    for (r = 0; r < 3; ++r) {
        if ((rc = one_round(r)) != 0) return rc;
        /* ends this process's context on the device; the next call runs in a new one */
        CK(cudaDeviceReset());
    }
    printf("ok\n");
    return 0;
}
"""


def test_static_scratch_after_context_reset(tmp_path):
    """A C host that allocates its own buffers, calls moe_layout and
    moe_layout_static, then destroys its context (cudaDeviceReset), three
    times: every round's layouts agree, so the scratch address used after a
    reset is the new context's, not the one remembered from before."""
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    _lib.load()                                   # builds the library if needed
    src = tmp_path / "reset_host.c"
    exe = tmp_path / "reset_host"
    src.write_text(C_RESET_HOST)
    cuda = os.environ.get("CUDA_HOME", "/usr/local/cuda")
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.join(root, "include"),
                    "-I", os.path.join(cuda, "include"), str(src), "-L", lib_dir, "-lmoe_layout",
                    "-L", os.path.join(cuda, "lib64"), "-lcudart", f"-Wl,-rpath,{lib_dir}",
                    f"-Wl,-rpath,{os.path.join(cuda, 'lib64')}", "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True, timeout=120)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)
