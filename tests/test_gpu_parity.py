"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Bit-exact: layout counts / offsets / row indices, dispatched bf16 rows, FP8
bytes and scales.  Combine: within one bf16 step (relative 2^-8); the
kernel's fp32 fused multiply-adds run in the oracle's order, so the
expected difference is zero and the count of differing elements is
reported.  Every workload, the prefill batch (M = 65536: 334k FP8 dispatch
rows, 65,536 combined tokens) included, is compared element by element: the
comparison runs in chunks, the oracle on the host's cores in parallel.
"""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import (POISON_BYTE, combine_all_tokens, compare_combine, compare_dispatch_rows,
                         compare_layout, dispatch_all_rows, problem_of, run_path, to_dev,
                         untouched_rows_ok)

pytestmark = pytest.mark.gpu
DEV = "cuda"

FULL = ["decode-M128-uniform", "M4096-zipf1.1", "M16384-hotpairs-dedup", "M8192-uniform-fp8"]


def _inputs(w, dev=DEV):
    d = W.make_inputs(w, device=dev)
    return d["topk_idx"], d["part_of"], d["topk_weights"], d["x"], d["y"]


def check_all(w, idx, po, gates, x, y, dev=DEV):
    prob = problem_of(w)
    ref = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    b = run_path(prob, idx, po, gates, x, y, dev)
    compare_layout(b, ref, prob)
    x_bits = oracle.bf16_bits(x)
    assert dispatch_all_rows(b, prob, x_bits, ref["disp_token"]) == ref["R_disp"]
    untouched_rows_ok(b, ref["R_disp"])
    n_diff = combine_all_tokens(b, y, gates, ref["exp_row"])
    return ref, b, n_diff


@pytest.mark.parametrize("name", FULL)
def test_workload_full_parity(name):
    w = W.get(name)
    ref, _, n_diff = check_all(w, *_inputs(w))
    assert ref["R_disp"] > 0
    assert n_diff == 0, f"{n_diff} combine elements off by one bf16 step"


def test_prefill_workload_full_parity():
    """The largest workload, every element: the whole layout, all R_disp FP8
    dispatch rows and their scales bit-exact, every combined token within one
    bf16 step (expected: identical), rows past R_disp untouched."""
    w = W.get("prefill-M65536-mix-dedup-fp8")
    ref, _, n_diff = check_all(w, *_inputs(w))
    assert ref["R_disp"] > 300_000
    assert n_diff == 0, f"{n_diff} combine elements off by one bf16 step"


# (M, N, G, topk, E, dedup, fp8, routing) -- ragged tails, odd sizes, extremes
SHAPES = [
    (1, 8, 1, 1, 1, False, False, "uniform"),
    (1, 128, 4, 2, 2, True, True, "uniform"),
    (37, 136, 10, 3, 4, False, False, "uniform"),
    (37, 136, 10, 3, 4, True, False, "zipf"),
    (1000, 256, 7, 7, 3, True, False, "uniform"),
    (257, 128, 64, 1, 64, True, True, "uniform"),
    (300, 512, 1024, 32, 64, True, False, "uniform"),
    (300, 512, 1024, 32, 64, False, True, "zipf"),
    (9473, 64, 256, 8, 8, True, False, "mix"),       # 148 * 64 + 1 tokens: ragged last tile
    (70001, 8, 256, 8, 8, True, False, "uniform"),   # many tiles, layout-heavy
    (4097, 384, 48, 6, 5, False, True, "zipf"),
    (2048, 7168, 256, 8, 8, True, True, "uniform"),
    (1024, 64, 256, 8, 8, True, False, "zipf"),      # 8192 pairs: largest one-cluster layout
    (1025, 64, 256, 8, 8, True, False, "zipf"),      # 8200 pairs: two-launch layout
    (16385, 64, 256, 8, 8, True, False, "zipf"),
    (310001, 8, 256, 8, 8, True, False, "uniform"),  # tiles too big for the id cache
]


@pytest.mark.parametrize("M,N,G,topk,E,dedup,fp8,routing", SHAPES)
def test_shapes(M, N, G, topk, E, dedup, fp8, routing):
    w = W.Workload(f"shape{M}", M=M, N=N, G=G, topk=topk, E_part=E, routing=routing,
                   placement="contiguous", dedup=dedup, fp8=fp8, zipf_s=1.1, seed=M + N)
    idx, po, gates, x, y = _inputs(w)
    # a shuffled placement so partitions hold non-contiguous experts
    po = np.random.default_rng(M).permutation(po).astype(np.int32)
    _, _, n_diff = check_all(w, idx, po, gates, x, y)
    assert n_diff == 0


def _custom(M, N, G, topk, E, dedup=False, fp8=False, seed=0):
    return W.Workload("custom", M=M, N=N, G=G, topk=topk, E_part=E, routing="uniform",
                      placement="contiguous", dedup=dedup, fp8=fp8, seed=seed)


@pytest.mark.parametrize("dedup", [False, True])
def test_degenerate_routing(dedup):
    w = _custom(2000, 256, 16, 4, 8, dedup=dedup)
    idx, po, gates, x, y = _inputs(w)
    # every token on one expert, in every slot (duplicates)
    check_all(w, np.full_like(idx, 5), po, gates, x, y)
    # duplicates inside tokens, and all experts on partition 0 (others empty)
    rng = np.random.default_rng(3)
    dup = rng.integers(0, 3, size=idx.shape).astype(np.int32)
    check_all(w, dup, np.zeros_like(po), gates, x, y)


@pytest.mark.parametrize("dedup", [False, True])
def test_invalid_ids_set_status(dedup):
    w = _custom(500, 128, 32, 4, 4, dedup=dedup, fp8=dedup)
    idx, po, gates, x, y = _inputs(w)
    idx = idx.copy()
    idx[7, 1] = -1
    idx[100, 3] = 32
    ref, b, _ = check_all(w, idx, po, gates, x, y)
    assert ref["status"] == moe.MOE_STATUS_BAD_EXPERT
    po2 = po.copy()
    po2[3] = 4                                        # placement entry out of range
    ref, b, _ = check_all(w, idx, po2, gates, x, y)
    assert ref["status"] == moe.MOE_STATUS_BAD_EXPERT | moe.MOE_STATUS_BAD_PART


def test_empty_batch():
    prob = moe.MoEProblem(0, 256, 16, 2, 4, True, True)
    b = moe.MoEBuffers(prob, DEV)
    b.layout.status.fill_(-1)
    b.layout_(torch.empty((0, 2), dtype=torch.int32, device=DEV),
              torch.zeros(16, dtype=torch.int32, device=DEV))
    b.dispatch_(torch.empty((0, 256), dtype=torch.bfloat16, device=DEV))
    b.combine_(torch.empty((0, 256), dtype=torch.bfloat16, device=DEV),
               torch.empty((0, 2), dtype=torch.float32, device=DEV))
    torch.cuda.synchronize()
    assert b.layout.status.item() == 0
    assert b.layout.part_offset.tolist() == [0] * 5
    assert b.layout.expert_offset.tolist() == [0] * 17


def test_fp8_every_bf16_value():
    """All finite bf16 values, blocked into rows, plus engineered blocks."""
    bits = np.arange(1 << 16, dtype=np.uint32).astype(np.uint16)
    f = oracle.bits_to_f32(bits)
    fin = bits[np.isfinite(f)]
    rng = np.random.default_rng(17)
    N = 1024
    M = (fin.size + N - 1) // N
    flat = np.concatenate([rng.permutation(fin), np.zeros(M * N - fin.size, np.uint16)])
    x = flat.reshape(M, N)
    extra = np.zeros((6, N), np.uint16)
    extra[0, :128] = 0x8000                                  # all -0
    extra[1, :128] = oracle.bf16_round(np.float32(rng.standard_normal(128)))
    extra[1, 5] = 0x8000                                     # -0 in a non-zero block
    extra[2, :128] = oracle.bf16_round(np.float32(np.arange(128) * 0.25 - 16))
    extra[2, 127] = oracle.bf16_round(np.float32([448.0]))[0]   # scale exactly 1: ties hit
    extra[3, :128] = oracle.bf16_round(np.float32(rng.standard_normal(128) * 2.0 ** -130))
    extra[4, :] = oracle.bf16_round(np.float32(rng.standard_normal(N) * 1e30))
    extra[5, 128:256] = oracle.bf16_round(np.float32(np.full(128, -3.0)))
    x = np.concatenate([x, extra])
    # sorted rows as well: blocks of similar magnitude exercise the subnormal range
    x = np.concatenate([x, np.sort(fin)[: (fin.size // N) * N].reshape(-1, N)])
    M = x.shape[0]
    G, topk, E = 8, 2, 4
    w = _custom(M, N, G, topk, E, dedup=False, fp8=True, seed=5)
    idx = W.make_routing(w)
    po = W.make_placement(w)
    gates = W.make_gates(w)
    xt = torch.from_numpy(x.view(np.int16)).to(DEV).view(torch.bfloat16)
    y = W.make_expert_outputs(w, device=DEV)
    prob = problem_of(w)
    ref = oracle.layout(idx, po, G, E, False)
    b = run_path(prob, idx, po, gates, xt, y)
    compare_layout(b, ref, prob)
    compare_dispatch_rows(b, prob, x, ref["disp_token"])


def test_layout_deterministic_and_reusable():
    w = W.get("M4096-zipf1.1").replace(N=64)
    idx, po, gates, x, y = _inputs(w)
    prob = problem_of(w)
    b = moe.MoEBuffers(prob, DEV)
    idx_d, po_d = to_dev(idx), to_dev(po)
    snaps = []
    for _ in range(3):
        b.layout_(idx_d, po_d)
        torch.cuda.synchronize()
        snaps.append([t.clone() for t in (b.layout.exp_row, b.layout.disp_token,
                                          b.layout.expert_offset, b.layout.part_offset)])
    for s in snaps[1:]:
        for a_, b_ in zip(snaps[0], s):
            assert torch.equal(a_, b_)


def test_binding_and_abi_reject_bad_calls():
    prob = moe.MoEProblem(64, 128, 8, 2, 2)
    b = moe.MoEBuffers(prob, DEV)
    idx = torch.zeros((64, 2), dtype=torch.int32, device=DEV)
    po = torch.zeros(8, dtype=torch.int32, device=DEV)
    with pytest.raises(TypeError):
        b.layout_(idx.long(), po)
    with pytest.raises(ValueError):
        b.layout_(idx.t(), po)
    with pytest.raises(moe.MoEError) as e:
        moe.moe_layout(prob, idx, po, b.layout, b.workspace[:16])
    assert e.value.code == 2
    bad = moe.MoEProblem(64, 120, 8, 2, 2, fp8=True)     # N % 128 != 0 with fp8
    with pytest.raises(moe.MoEError) as e:
        moe.moe_layout(bad, idx, po, b.layout, b.workspace)
    assert e.value.code == 1
    torch.cuda.synchronize()


def test_streams_and_graph_capture():
    """The three calls are stream-ordered and capturable in a CUDA graph."""
    w = W.get("M4096-zipf1.1").replace(M=1024, N=512)
    idx, po, gates, x, y = _inputs(w)
    prob = problem_of(w)
    b = moe.MoEBuffers(prob, DEV)
    idx_d, po_d, g_d = to_dev(idx), to_dev(po), to_dev(gates)
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        b.step(idx_d, po_d, x, y, g_d)
    s.synchronize()
    out_eager = b.out.clone()
    b.out.zero_()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        b.step(idx_d, po_d, x, y, g_d)
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(b.out, out_eager)
    ref = oracle.layout(idx, po, w.G, w.E_part, False)
    compare_combine(b, prob, y, gates, ref["exp_row"])
    del g


@pytest.mark.parametrize("fp8,dedup", [(False, False), (True, True)])
def test_buffers_only_16_byte_aligned(fp8, dedup):
    """Rows that allow 32-byte vectors but buffers that start 16 bytes past a
    32-byte boundary take the 16-byte paths; results are the same."""
    w = _custom(777, 1024, 64, 6, 8, dedup=dedup, fp8=fp8, seed=9)
    idx, po, gates, x0, y0 = _inputs(w)
    prob = problem_of(w)

    def shifted(t):
        off = 16 // t.element_size()               # 16 bytes, whatever the dtype
        flat = torch.empty(t.numel() + off, dtype=t.dtype, device=t.device)
        v = flat[off:].view(t.shape)
        v.copy_(t)
        assert v.data_ptr() % 32 == 16
        return v

    x, y = shifted(x0), shifted(y0)
    b = moe.MoEBuffers(prob, DEV)
    b.recv_x = shifted(b.recv_x.view(torch.uint8 if fp8 else torch.bfloat16))
    b.out = shifted(b.out)
    b.layout_(to_dev(idx), to_dev(po))
    b.dispatch_(x)
    b.combine_(y, to_dev(gates))
    torch.cuda.synchronize()
    ref = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    compare_dispatch_rows(b, prob, oracle.bf16_bits(x0), ref["disp_token"])
    assert compare_combine(b, prob, y0, gates, ref["exp_row"]) == 0
