"""The expert-parallel data plane (moe_ep_dispatch, moe_ep_combine,
moe_ep_combine_reduce) on one GPU with W ranks emulated by W sets of
buffers: every source pushes its rows into all W receive buffers through a
table of device pointers, at the offsets of its moe_ep_plan; then every
source pulls its tokens' outputs back from per-rank buffers.  Checked
against the oracle: each receive buffer holds, in source-rank order, every
source's dispatch rows for it (bytes and FP8 scales bit-exact, rows past the
filled range untouched), and each combine equals the oracle's combine (or
token-side reduce) over the rows gathered from the ranks' buffers.  No
kernel waits on another: the ranks' kernels run one after another."""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W
from gpu_harness import POISON_BYTE, ulp_distance_bf16

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _world(world, M, N, G, topk, dedup, fp8, seed):
    ranks = []
    for s in range(world):
        w = W.Workload("ep", M=M + 5 * s, N=N, G=G, topk=topk, E_part=world, routing="mix",
                       placement="contiguous", dedup=dedup, fp8=fp8, seed=seed + s)
        d = W.make_inputs(w, device=DEV, with_y=False)
        prob = moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)
        lay = moe.alloc_layout(prob, DEV)
        ws = torch.empty(moe.layout_workspace_size(prob), dtype=torch.uint8, device=DEV)
        idx, po = torch.from_numpy(d["topk_idx"]).to(DEV), torch.from_numpy(d["part_of"]).to(DEV)
        moe.moe_layout(prob, idx, po, lay, ws)
        ranks.append(dict(w=w, d=d, prob=prob, lay=lay, ws=ws))
    torch.cuda.synchronize()
    P = torch.stack([r["lay"].part_count for r in ranks])
    for s, r in enumerate(ranks):
        r["plan"] = moe.alloc_ep_plan(world, 0, DEV)
        moe.moe_ep_plan(world, s, P, r["plan"])
    torch.cuda.synchronize()
    for r in ranks:
        r["ref"] = oracle.layout(r["d"]["topk_idx"], r["d"]["part_of"], r["w"].G, world, dedup)
        r["so"] = r["plan"].send_offset.cpu().numpy()
        r["po"] = r["ref"]["part_offset"]
    return ranks


def _gathered(ranks, s, bufs):
    """Rows of source s's dispatch space, gathered from the ranks' buffers
    at its plan's offsets (host copy, bf16 bits)."""
    r = ranks[s]
    R = int(r["po"][-1])
    out = np.zeros((max(R, 1), bufs[0].shape[1]), np.uint16)
    for p in range(len(ranks)):
        a, b = int(r["po"][p]), int(r["po"][p + 1])
        o = int(r["so"][p])
        out[a:b] = oracle.bf16_bits(bufs[p][o:o + b - a])
    return out[:R]


CASES = [  # world, M, N, G, topk, dedup, fp8
    (1, 40, 128, 8, 2, False, False),
    (2, 300, 256, 32, 4, False, False),
    (4, 500, 128, 64, 8, False, True),
    (8, 1000, 1024, 256, 8, False, False),
    (3, 400, 256, 48, 6, True, False),
    (8, 700, 512, 256, 8, True, True),
]


@pytest.mark.parametrize("world,M,N,G,topk,dedup,fp8", CASES)
def test_push_dispatch_and_pull_combine(world, M, N, G, topk, dedup, fp8):
    ranks = _world(world, M, N, G, topk, dedup, fp8, seed=M + world)
    totals = [int(r["plan"].recv_offset[world].item()) for r in ranks]
    cap = max(totals) + 3                              # slack rows must stay untouched
    row_dtype = torch.uint8 if fp8 else torch.bfloat16
    recv = [torch.full((cap, N), 0, dtype=row_dtype, device=DEV) for _ in range(world)]
    for t in recv:
        t.view(torch.uint8).fill_(POISON_BYTE)
    scale = [torch.full((cap, N // 128), 0.0, device=DEV) for _ in range(world)] if fp8 else None
    if fp8:
        for t in scale:
            t.view(torch.uint8).fill_(POISON_BYTE)
    peers = moe.ep_peers(recv, cap, scale, DEV)
    for r in ranks:
        moe.moe_ep_dispatch(r["prob"], r["d"]["x"], r["lay"], r["plan"].send_offset, peers)
    torch.cuda.synchronize()
    for r in ranks:
        assert r["lay"].status.item() == 0
    # each receive buffer: every source's rows for it, in source order
    for d_ in range(world):
        for s, r in enumerate(ranks):
            a, b = int(r["po"][d_]), int(r["po"][d_ + 1])
            o = int(ranks[s]["so"][d_])
            toks = r["ref"]["disp_token"][a:b]
            xb = oracle.bf16_bits(r["d"]["x"])
            if fp8:
                q, sc = oracle.dispatch(xb, toks, True)
                np.testing.assert_array_equal(recv[d_][o:o + b - a].cpu().numpy(), q)
                np.testing.assert_array_equal(scale[d_][o:o + b - a].cpu().numpy().view(np.uint32),
                                              sc.view(np.uint32))
            else:
                np.testing.assert_array_equal(oracle.bf16_bits(recv[d_][o:o + b - a]),
                                              oracle.dispatch(xb, toks, False))
        assert bool((recv[d_][totals[d_]:].view(torch.uint8) == POISON_BYTE).all())
    # the return trip: outputs computed by each destination in its receive order
    g = torch.Generator(device=DEV)
    g.manual_seed(world * 1000 + M)
    outs = [torch.randn((cap, N), generator=g, device=DEV).to(torch.bfloat16) for _ in range(world)]
    out_peers = moe.ep_peers(outs, cap, device=DEV)
    for s, r in enumerate(ranks):
        out = torch.empty((r["w"].M, N), dtype=torch.bfloat16, device=DEV)
        gates = torch.from_numpy(r["d"]["topk_weights"]).to(DEV)
        if dedup:
            moe.moe_ep_combine_reduce(r["prob"], out_peers, r["lay"], r["plan"].send_offset, out)
        else:
            moe.moe_ep_combine(r["prob"], out_peers, gates, r["lay"], r["plan"].send_offset, out)
        torch.cuda.synchronize()
        assert r["lay"].status.item() == 0
        rows = _gathered(ranks, s, outs)
        if dedup:
            want = oracle.combine_reduce(rows, r["ref"]["disp_row"])
        else:
            want = oracle.combine(rows, r["d"]["topk_weights"], r["ref"]["exp_row"])
        got = oracle.bf16_bits(out)
        assert ulp_distance_bf16(got, want).max(initial=0) <= 1
        assert np.count_nonzero(got != want) == 0


def test_same_bytes_as_the_local_dispatch():
    """With one rank the exchange is the local dispatch: same bytes."""
    ranks = _world(1, 777, 1024, 64, 6, True, True, seed=3)
    r = ranks[0]
    cap = r["prob"].capacity
    recv = torch.empty((cap, 1024), dtype=torch.uint8, device=DEV)
    sc = torch.empty((cap, 8), dtype=torch.float32, device=DEV)
    moe.moe_ep_dispatch(r["prob"], r["d"]["x"], r["lay"], r["plan"].send_offset,
                        moe.ep_peers([recv], cap, [sc], DEV))
    local = torch.empty_like(recv)
    lsc = torch.empty_like(sc)
    moe.moe_dispatch(r["prob"], r["d"]["x"], r["lay"], local, lsc)
    torch.cuda.synchronize()
    R = int(r["po"][-1])
    assert torch.equal(recv[:R], local[:R]) and torch.equal(sc[:R].view(torch.int32),
                                                            lsc[:R].view(torch.int32))


def test_rows_outside_a_buffer_are_skipped_and_flagged():
    ranks = _world(2, 200, 128, 16, 4, False, False, seed=9)
    totals = [int(r["plan"].recv_offset[2].item()) for r in ranks]
    cap = min(totals) // 2                             # too small for either destination
    # each buffer is the head of a larger poisoned one: nothing may land past cap
    big = [torch.empty((cap + 64, 128), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    for t in big:
        t.view(torch.uint8).fill_(POISON_BYTE)
    recv = [t[:cap] for t in big]
    peers = moe.ep_peers(recv, cap, device=DEV)
    for r in ranks:
        r["lay"].status.zero_()
        moe.moe_ep_dispatch(r["prob"], r["d"]["x"], r["lay"], r["plan"].send_offset, peers)
    torch.cuda.synchronize()
    assert all(r["lay"].status.item() & moe.MOE_STATUS_BAD_ROW for r in ranks)
    for t in big:
        assert bool((t[cap:].view(torch.uint8) == POISON_BYTE).all())
    # a misaligned pointer in the table: that rank's rows are skipped
    bad = moe.ep_peers([recv[0].data_ptr() + 2, recv[1]], cap, device=DEV)
    r = ranks[0]
    r["lay"].status.zero_()
    before = recv[0].clone()
    moe.moe_ep_dispatch(r["prob"], r["d"]["x"], r["lay"], r["plan"].send_offset, bad)
    torch.cuda.synchronize()
    assert r["lay"].status.item() & moe.MOE_STATUS_BAD_ROW
    assert torch.equal(recv[0], before)


def test_arguments_are_checked_on_the_host():
    ranks = _world(2, 50, 128, 8, 2, False, False, seed=1)
    r = ranks[0]
    recv = [torch.empty((100, 128), dtype=torch.bfloat16, device=DEV) for _ in range(2)]
    with pytest.raises(ValueError):                   # one buffer per partition
        moe.moe_ep_dispatch(r["prob"], r["d"]["x"], r["lay"], r["plan"].send_offset,
                            moe.ep_peers(recv[:1], 100, device=DEV))
    with pytest.raises(ValueError):                   # a combine of a dedup layout
        moe.moe_ep_combine_reduce(r["prob"], moe.ep_peers(recv, 100, device=DEV), r["lay"],
                                  r["plan"].send_offset, recv[0][:50])
