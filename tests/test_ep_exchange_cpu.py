"""The expert-parallel counts exchange and the data exchange it plans, as
real processes on CPU (gloo): W ranks each route their own tokens over
partitions = ranks, gather every rank's counts with the binding's
ep_all_gather_counts, take their plan (the oracle's, on CPU), and move their
dispatch rows with torch.distributed.all_to_all_single at those splits.
Each destination must then hold, in source-rank order, exactly every
source's rows for it (Purlin section 3.1, transposed-V layout), every
rank's push offsets must be the destinations' receive offsets, and the
reverse exchange (the combine's return trip) must give every source its
rows back in its own dispatch order."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import workloads as W

BIG = 1 << 20


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, dedup, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import combine_moe_layout_08_b200 as moe
        import oracle
        w = W.Workload("ep", M=61 + 17 * rank, N=16, G=24, topk=4, E_part=world,
                       routing="zipf", placement="contiguous", dedup=dedup, seed=10 + rank)
        idx, po = W.make_routing(w), W.make_placement(w)
        lay = oracle.layout(idx, po, w.G, world, dedup)
        # the counts exchange through the binding (gloo on CPU tensors)
        P = moe.ep_all_gather_counts(torch.from_numpy(lay["part_count"].copy()))
        X = moe.ep_all_gather_counts(torch.from_numpy(lay["expert_count"].copy()))
        assert P.shape == (world, world) and X.shape == (world, w.G)
        plan = oracle.ep_plan(P.numpy(), rank, None if dedup else X.numpy(),
                              None if dedup else po)
        assert plan["status"] == 0
        # dispatch rows as (source, token) payloads, in this rank's dispatch order
        send = torch.from_numpy(rank * BIG + lay["disp_token"].astype(np.int64))
        recv = torch.empty(int(plan["recv_offset"][world]), dtype=torch.int64)
        dist.all_to_all_single(recv, send, output_split_sizes=plan["recv_count"].tolist(),
                               input_split_sizes=P[rank].tolist())
        # the return trip: every destination sends its rows back to their sources
        back = torch.empty_like(send)
        dist.all_to_all_single(back, recv, output_split_sizes=P[rank].tolist(),
                               input_split_sizes=plan["recv_count"].tolist())
        everyone = [None] * world
        dist.all_gather_object(everyone, dict(disp_token=lay["disp_token"].tolist(),
                                              part_offset=lay["part_offset"].tolist(),
                                              expert_offset=lay["expert_offset"].tolist(),
                                              expert_count=lay["expert_count"].tolist(),
                                              plan={k: np.asarray(v).tolist()
                                                    for k, v in plan.items() if k != "status"}))
        q.put((rank, recv.tolist(), torch.equal(back, send), everyone))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,dedup", [(2, False), (2, True), (3, False)])
def test_exchange_over_gloo_ranks(world, dedup):
    port = _free_port()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    procs = [ctx.Process(target=_worker, args=(r, world, port, dedup, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=180) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    everyone = res[0][3]
    for r, recv, back_ok, _ in res:
        assert back_ok, f"rank {r}: the return trip did not restore its rows"
        # by definition: source order, each source's rows of partition r
        want = []
        for s, e in enumerate(everyone):
            a, b = e["part_offset"][r], e["part_offset"][r + 1]
            want += [s * BIG + t for t in e["disp_token"][a:b]]
        assert recv == want, f"rank {r}: receive buffer is not the transposed-V layout"
        pl = everyone[r]["plan"]
        for s in range(world):
            # push offset of s towards r == r's receive offset of s
            assert everyone[s]["plan"]["send_offset"][r] == pl["recv_offset"][s]
            # pull offset == where s's rows for r start in s's own dispatch order
            assert pl["src_offset"][s] == everyone[s]["part_offset"][r]
        if not dedup:
            blk = np.array(pl["recv_block_offset"])
            for s, e in enumerate(everyone):
                for g in np.flatnonzero(blk[s] >= 0):
                    o, n, a = blk[s][g], e["expert_count"][g], e["expert_offset"][g]
                    # the block holds source s's expert rows of g
                    assert recv[o:o + n] == [s * BIG + t for t in e["disp_token"][a:a + n]]
