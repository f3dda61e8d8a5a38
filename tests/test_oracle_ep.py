"""Pins of the oracle's expert-parallel exchange plan (oracle.ep_plan).

The plan turns every rank's per-partition row counts (and, without dedup,
per-expert counts) into offsets: the counts exchange of the Triton-
distributed issue #117 all-to-all (split_send_buf -> split_recv_buf,
send_split_cumsum), into Purlin's transposed-V layout (section 3.1:
destination r receives partition r from every source and arranges it in
source-rank order).  The pins do not retype the plan's sums.  They simulate
the exchange on W ranks whose layouts come from oracle.layout over their own
tokens, and build every receive buffer three ways:
  * by the definition: the concatenation, in source order, of each source's
    rows of partition r, cut out with that source's own layout offsets;
  * by pushes: every source writes its rows at the plan's send offsets, and
    every destination slot is written exactly once;
  * by pulls: every destination reads each source's rows at the plan's
    source offsets.
Expert blocks are checked against each source's expert rows, and a few
closed forms and the status word close the list."""
import numpy as np
import pytest

import oracle

BIG = 1 << 20


def _ranks(W, seed, G, topk, dedup, M_max=40):
    rng = np.random.default_rng(seed)
    po = rng.integers(0, W, size=G).astype(np.int32)
    ranks = []
    for s in range(W):
        M = int(rng.integers(0, M_max))
        idx = np.stack([rng.choice(G, size=topk, replace=False) for _ in range(M)]).astype(np.int32) \
            if M else np.zeros((0, topk), np.int32)
        lay = oracle.layout(idx, po, G, W, dedup)
        # payload of a dispatch row: (source rank, token), so rows are traceable
        lay["payload"] = s * BIG + lay["disp_token"].astype(np.int64)
        ranks.append(lay)
    return po, ranks


def _counts(ranks):
    P = np.stack([r["part_count"] for r in ranks]).astype(np.int32)
    X = np.stack([r["expert_count"] for r in ranks]).astype(np.int32)
    return P, X


CASES = [(1, 0, 4, 2), (2, 1, 8, 3), (3, 2, 12, 2), (4, 3, 16, 4), (8, 4, 32, 8), (5, 5, 7, 1)]


@pytest.mark.parametrize("W,seed,G,topk", CASES)
@pytest.mark.parametrize("dedup", [False, True])
def test_exchange_by_definition_push_and_pull(W, seed, G, topk, dedup):
    po, ranks = _ranks(W, seed, G, topk, dedup)
    P, X = _counts(ranks)
    plans = [oracle.ep_plan(P, r) for r in range(W)]
    assert all(p["status"] == 0 for p in plans)
    # the definition: source order, each source's partition-r rows
    want = [np.concatenate([ranks[s]["payload"][ranks[s]["part_offset"][r]:
                                                 ranks[s]["part_offset"][r + 1]]
                            for s in range(W)]) for r in range(W)]
    for r in range(W):
        assert plans[r]["recv_offset"][W] == want[r].size
        np.testing.assert_array_equal(plans[r]["recv_count"], P[:, r])
    # pushes: source s writes its rows for d at its own send offset in d's buffer
    pushed = [np.full(w.size, -1, np.int64) for w in want]
    writes = [np.zeros(w.size, np.int64) for w in want]
    for s in range(W):
        for d in range(W):
            a = ranks[s]["part_offset"][d]
            n = int(P[s, d])
            o = plans[s]["send_offset"][d]
            assert 0 <= o and o + n <= pushed[d].size, "push outside the receive buffer"
            pushed[d][o:o + n] = ranks[s]["payload"][a:a + n]
            writes[d][o:o + n] += 1
    # pulls: destination r reads each source's rows at the plan's source offsets
    pulled = [np.full(w.size, -1, np.int64) for w in want]
    for r in range(W):
        pl = plans[r]
        for s in range(W):
            o, n, a = pl["recv_offset"][s], pl["recv_count"][s], pl["src_offset"][s]
            assert 0 <= o and o + n <= pulled[r].size, "pull outside the receive buffer"
            assert 0 <= a and a + n <= ranks[s]["payload"].size, "pull outside the source rows"
            pulled[r][o:o + n] = ranks[s]["payload"][a:a + n]
    for r in range(W):
        assert np.all(writes[r] == 1), "every receive slot written exactly once"
        np.testing.assert_array_equal(pushed[r], want[r])
        np.testing.assert_array_equal(pulled[r], want[r])


@pytest.mark.parametrize("W,seed,G,topk", CASES)
def test_expert_blocks_hold_each_sources_expert_rows(W, seed, G, topk):
    po, ranks = _ranks(W, seed + 100, G, topk, False)
    P, X = _counts(ranks)
    for r in range(W):
        pl = oracle.ep_plan(P, r, X, po)
        assert pl["status"] == 0
        recv = np.concatenate([ranks[s]["payload"][ranks[s]["part_offset"][r]:
                                                   ranks[s]["part_offset"][r + 1]]
                               for s in range(W)])
        cover = np.zeros(recv.size, np.int64)
        for e in range(G):
            if po[e] != r:
                assert pl["recv_expert_count"][e] == 0
                assert np.all(pl["recv_block_offset"][:, e] == -1)
                continue
            assert pl["recv_expert_count"][e] == X[:, e].sum()
            for s in range(W):
                o, n = pl["recv_block_offset"][s, e], X[s, e]
                a = ranks[s]["expert_offset"][e]
                assert 0 <= o and o + n <= recv.size, "block outside the receive buffer"
                # the block holds exactly source s's expert rows of e (no dedup:
                # dispatch rows are expert rows)
                np.testing.assert_array_equal(recv[o:o + n], ranks[s]["payload"][a:a + n])
                cover[o:o + n] += 1
        assert np.all(cover == 1), "the (source, expert) blocks tile the receive buffer"


def test_closed_forms():
    # one rank: everything starts at 0 and it receives its own rows
    pl = oracle.ep_plan(np.array([[7]]), 0)
    assert list(pl["send_offset"]) == [0] and list(pl["src_offset"]) == [0]
    assert list(pl["recv_offset"]) == [0, 7]
    # every rank sends c rows to every rank: offsets are multiples of c
    W, c = 6, 5
    P = np.full((W, W), c)
    for r in range(W):
        pl = oracle.ep_plan(P, r)
        assert list(pl["send_offset"]) == [r * c] * W
        assert list(pl["src_offset"]) == [r * c] * W
        assert list(pl["recv_offset"]) == [s * c for s in range(W + 1)]
    # an upper-triangular send pattern
    P = np.triu(np.arange(1, 17).reshape(4, 4))
    pl = oracle.ep_plan(P, 2)                                 # rows 0 and 1 precede rank 2
    assert list(pl["send_offset"]) == [1 + 0, 2 + 6, 3 + 7, 4 + 8]
    assert list(pl["src_offset"]) == [1 + 2, 0 + 6, 0, 0]
    assert list(pl["recv_offset"]) == [0, 3, 3 + 7, 3 + 7 + 11, 3 + 7 + 11]


def test_status_flags_bad_counts():
    assert oracle.ep_plan(np.array([[1, -1], [0, 2]]), 0)["status"] == 8
    big = np.full((3, 3), 1 << 30, np.int32)                  # sums past 2^31 - 1
    pl = oracle.ep_plan(big, 2)
    assert pl["status"] == 8 and -1 in pl["send_offset"] and pl["recv_offset"][3] == -1
    # expert counts that do not add up to the partition counts
    P = np.array([[2, 1], [0, 3]])
    X = np.array([[2, 0, 1], [0, 2, 0]])                      # rank 1's rows to 1: 2 != 3
    po = np.array([0, 1, 1])
    assert oracle.ep_plan(P, 1, X, po)["status"] == 8
    X[1, 2] = 1
    assert oracle.ep_plan(P, 1, X, po)["status"] == 0
