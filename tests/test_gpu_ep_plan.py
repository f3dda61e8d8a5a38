"""moe_ep_plan on the GPU against the oracle, with W ranks emulated on one
GPU: W layouts of W token batches (one per rank, partitions = ranks), their
counts stacked as the counts exchange would give them, then every rank's
plan bit-exact against oracle.ep_plan.  The data exchange the plan drives is
emulated with device copies at the plan's offsets (pulls: each destination
reads every source's rows at src_offset): each receive buffer must hold
every source's rows for it in source-rank order, each (source, expert) block
the source's rows of that expert, and the pushes (send_offset) must land in
the same places."""
import numpy as np
import pytest
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _ranks(world, M, N, G, topk, dedup, seed):
    out = []
    for s in range(world):
        w = W.Workload("ep", M=M + 7 * s, N=N, G=G, topk=topk, E_part=world, routing="zipf",
                       placement="contiguous", dedup=dedup, seed=seed + s)
        d = W.make_inputs(w, device=DEV, with_y=False)
        prob = moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)
        b = moe.MoEBuffers(prob, DEV)
        idx, po = torch.from_numpy(d["topk_idx"]).to(DEV), torch.from_numpy(d["part_of"]).to(DEV)
        b.layout_(idx, po)
        b.dispatch_(d["x"])
        out.append((w, d, b, po))
    torch.cuda.synchronize()
    return out


@pytest.mark.parametrize("world,M,N,G,topk,dedup", [
    (1, 50, 64, 16, 4, False), (2, 300, 128, 32, 4, False), (4, 1000, 64, 64, 8, False),
    (8, 4096, 256, 256, 8, False), (8, 2000, 64, 256, 8, True), (3, 700, 64, 48, 6, True),
    (64, 200, 64, 1024, 16, False),
])
def test_plan_matches_oracle_and_drives_the_exchange(world, M, N, G, topk, dedup):
    ranks = _ranks(world, M, N, G, topk, dedup, seed=M + world)
    P = torch.stack([b.layout.part_count for _, _, b, _ in ranks])
    X = torch.stack([b.layout.expert_count for _, _, b, _ in ranks])
    po = ranks[0][3]
    P_h, X_h, po_h = P.cpu().numpy(), X.cpu().numpy(), po.cpu().numpy()
    with_x = not dedup
    plans = []
    for r in range(world):
        plan = moe.alloc_ep_plan(world, G if with_x else 0, DEV)
        for t in (plan.send_offset, plan.src_offset, plan.recv_count, plan.recv_offset, plan.status):
            t.fill_(-7)
        moe.moe_ep_plan(world, r, P, plan, X if with_x else None, po if with_x else None)
        plans.append(plan)
    torch.cuda.synchronize()
    for r, plan in enumerate(plans):
        ref = oracle.ep_plan(P_h, r, X_h if with_x else None, po_h if with_x else None)
        assert plan.status.item() == ref["status"] == 0
        for k in ("send_offset", "src_offset", "recv_count", "recv_offset") + \
                (("recv_expert_count", "recv_block_offset") if with_x else ()):
            np.testing.assert_array_equal(getattr(plan, k).cpu().numpy(), ref[k], err_msg=k)
    # the exchange, emulated: pulls into each destination's receive buffer
    host = [(b.layout.part_offset.cpu().tolist(), b.layout.expert_offset.cpu().numpy(),
             b.layout.expert_count.cpu().numpy()) for _, _, b, _ in ranks]
    check = range(world) if world <= 8 else (0, world // 2, world - 1)
    for r in check:
        plan = plans[r]
        ro = plan.recv_offset.cpu().tolist()
        so = plan.src_offset.cpu().tolist()
        rc = plan.recv_count.cpu().tolist()
        recv = torch.empty((ro[world], N), dtype=torch.bfloat16, device=DEV)
        want = []
        for s, (_, _, b, _) in enumerate(ranks):
            recv[ro[s]:ro[s] + rc[s]] = b.recv_x[so[s]:so[s] + rc[s]]
            po_s = host[s][0]
            want.append(b.recv_x[po_s[r]:po_s[r + 1]])
        assert torch.equal(recv, torch.cat(want)), f"rank {r}: not the transposed-V layout"
        # pushes land in the same places
        for s in range(world):
            assert plans[s].send_offset[r].item() == ro[s]
        if with_x:
            blk = plan.recv_block_offset.cpu().numpy()
            for s, (_, _, b, _) in enumerate(ranks):
                _, eo, ec = host[s]
                for e in np.flatnonzero(po_h == r):
                    o, n, a = int(blk[s, e]), int(ec[e]), int(eo[e])
                    assert torch.equal(recv[o:o + n], b.recv_x[a:a + n]), (r, s, e)


def test_plan_flags_bad_counts_and_rejects_bad_arguments():
    P = torch.tensor([[1, -1], [0, 2]], dtype=torch.int32, device=DEV)
    plan = moe.alloc_ep_plan(2, 0, DEV)
    moe.moe_ep_plan(2, 0, P, plan)
    torch.cuda.synchronize()
    assert plan.status.item() == moe.MOE_STATUS_BAD_COUNT
    big = torch.full((3, 3), 1 << 30, dtype=torch.int32, device=DEV)
    plan3 = moe.alloc_ep_plan(3, 0, DEV)
    moe.moe_ep_plan(3, 2, big, plan3)
    torch.cuda.synchronize()
    ref = oracle.ep_plan(big.cpu().numpy(), 2)
    assert plan3.status.item() == ref["status"] == moe.MOE_STATUS_BAD_COUNT
    np.testing.assert_array_equal(plan3.send_offset.cpu().numpy(), ref["send_offset"])
    np.testing.assert_array_equal(plan3.recv_offset.cpu().numpy(), ref["recv_offset"])
    # expert counts that do not add up to the partition counts
    P2 = torch.tensor([[2, 1], [0, 3]], dtype=torch.int32, device=DEV)
    X2 = torch.tensor([[2, 0, 1], [0, 2, 0]], dtype=torch.int32, device=DEV)
    po2 = torch.tensor([0, 1, 1], dtype=torch.int32, device=DEV)
    plan2 = moe.alloc_ep_plan(2, 3, DEV)
    moe.moe_ep_plan(2, 1, P2, plan2, X2, po2)
    torch.cuda.synchronize()
    assert plan2.status.item() == moe.MOE_STATUS_BAD_COUNT
    with pytest.raises(moe.MoEError) as e:
        moe.moe_ep_plan(2, 2, P2, plan2)                         # rank out of range
    assert e.value.code == 1
