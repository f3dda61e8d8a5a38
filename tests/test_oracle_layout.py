"""Pins of the oracle's routing layout (CPU only).

* brute force: every top-k assignment and every placement map of tiny
  problems, against the rank-counting statement in ``layout_defs``;
* a second formulation at workload sizes: numpy ``lexsort`` over (p, e, t, k);
* invariants: counts sum to the number of valid pairs (or to the distinct
  (token, partition) pairs under dedup), offsets are monotone prefix sums,
  every pair appears exactly once, the maps are mutual inverses, rows of one
  expert / partition are in token order.
"""
import itertools

import numpy as np
import pytest

import oracle
import workloads as W
from layout_defs import py_layout


def _cmp(o, ref, dedup):
    assert o["status"] == ref["status"]
    assert o["R_exp"] == ref["R_exp"]
    assert o["R_disp"] == ref["R_disp"]
    assert o["expert_count"].tolist() == ref["expert_count"]
    assert o["expert_offset"].tolist() == ref["expert_offset"]
    assert o["part_count"].tolist() == ref["part_count"]
    assert o["part_offset"].tolist() == ref["part_offset"]
    assert o["exp_row"].tolist() == ref["exp_row"]
    assert o["disp_token"].tolist() == ref["disp_token"]
    if dedup:
        assert o["disp_row"].tolist() == ref["disp_row"]
        assert o["exp_to_disp"].tolist() == ref["exp_to_disp"]


# (M, topk, G, E_part, alphabet extra values)
EXHAUSTIVE = [
    (1, 1, 3, 2, ()),
    (2, 1, 3, 3, ()),
    (1, 3, 4, 2, ()),
    (2, 2, 3, 2, ()),
    (3, 2, 3, 2, ()),
    (3, 1, 4, 3, ()),
    (2, 2, 2, 2, (-1, 2)),      # invalid expert ids mixed in
]


@pytest.mark.parametrize("M,topk,G,E,extra", EXHAUSTIVE)
@pytest.mark.parametrize("dedup", [False, True])
def test_layout_exhaustive_tiny(M, topk, G, E, extra, dedup):
    alphabet = list(range(G)) + list(extra)
    placements = list(itertools.product(range(E), repeat=G))
    n_cases = 0
    for flat in itertools.product(alphabet, repeat=M * topk):
        idx = [list(flat[t * topk:(t + 1) * topk]) for t in range(M)]
        # every placement for small alphabets, a seeded third otherwise
        pl = placements if len(placements) <= 16 else placements[::3]
        for po in pl:
            o = oracle.layout(np.array(idx, np.int32).reshape(M, topk),
                              np.array(po, np.int32), G, E, dedup)
            _cmp(o, py_layout(idx, list(po), G, E, dedup), dedup)
            n_cases += 1
    assert n_cases > 0


@pytest.mark.parametrize("dedup", [False, True])
def test_layout_bad_placement_entries(dedup):
    rng = np.random.default_rng(7)
    G, E = 5, 3
    for _ in range(200):
        M, topk = int(rng.integers(1, 5)), int(rng.integers(1, 4))
        idx = rng.integers(-1, G + 1, size=(M, topk))
        po = rng.integers(-1, E + 1, size=G)
        o = oracle.layout(idx.astype(np.int32), po.astype(np.int32), G, E, dedup)
        _cmp(o, py_layout(idx.tolist(), po.tolist(), G, E, dedup), dedup)


def _random_problem(rng, M, topk, G, E, distinct=True):
    if distinct and topk <= G:
        idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk]
    else:
        idx = rng.integers(0, G, size=(M, topk))
    po = rng.integers(0, E, size=G)
    return idx.astype(np.int32), po.astype(np.int32)


def _check_invariants(idx, po, G, E, dedup, o):
    M, topk = idx.shape
    n = M * topk
    assert o["status"] == 0
    # counts
    assert o["expert_count"].sum() == n == o["R_exp"]
    np.testing.assert_array_equal(o["expert_count"], np.bincount(idx.ravel(), minlength=G))
    # expert-row space: a permutation of 0..n-1
    er = o["exp_row"].ravel()
    assert np.array_equal(np.sort(er), np.arange(n))
    # rows of expert e are the block [offset, offset + count), in (t, k) order
    for e in range(G):
        rows = er[idx.ravel() == e]
        off, cnt = o["expert_offset"][e], o["expert_count"][e]
        assert np.array_equal(rows, np.arange(off, off + cnt))
    # experts of one partition are contiguous and ordered by id
    order = sorted(range(G), key=lambda e: (po[e], e))
    starts = [o["expert_offset"][e] for e in order]
    assert starts == sorted(starts)
    # partitions
    po_ = o["part_offset"]
    assert po_[0] == 0 and np.all(np.diff(po_) == o["part_count"])
    if not dedup:
        assert o["R_disp"] == n
        tok = np.repeat(np.arange(M), topk)
        np.testing.assert_array_equal(o["disp_token"][er], tok)
        for p in range(E):
            assert o["part_count"][p] == o["expert_count"][po == p].sum()
    else:
        pairs = {(t, int(po[e])) for t in range(M) for e in idx[t]}
        assert o["R_disp"] == len(pairs) == o["part_count"].sum()
        dr = o["disp_row"]
        for t in range(M):
            want = {int(po[e]) for e in idx[t]}
            got = {p for p in range(E) if dr[t, p] >= 0}
            assert want == got
        valid = dr[dr >= 0]
        assert np.array_equal(np.sort(valid), np.arange(o["R_disp"]))
        # rows of partition p: tokens ascending
        for p in range(E):
            rows = dr[:, p][dr[:, p] >= 0]
            assert np.array_equal(rows, np.arange(po_[p], po_[p + 1]))
            assert np.all(np.diff(o["disp_token"][rows]) > 0)
        # exp_to_disp: the dispatch row of the expert row's (token, partition)
        tk = np.repeat(np.arange(M), topk)
        pp = po[idx.ravel()]
        np.testing.assert_array_equal(o["exp_to_disp"][er], dr[tk, pp])
        np.testing.assert_array_equal(o["disp_token"][o["exp_to_disp"][er]], tk)


@pytest.mark.parametrize("dedup", [False, True])
@pytest.mark.parametrize("M,topk,G,E", [(1, 1, 1, 1), (37, 3, 10, 4), (200, 8, 64, 8),
                                        (513, 2, 128, 8), (96, 6, 7, 3), (64, 4, 16, 64)])
def test_layout_invariants(M, topk, G, E, dedup):
    rng = np.random.default_rng(M * 1000 + G)
    idx, po = _random_problem(rng, M, topk, G, E)
    _check_invariants(idx, po, G, E, dedup, oracle.layout(idx, po, G, E, dedup))
    # duplicate expert ids inside one token
    idx2, _ = _random_problem(rng, M, topk, G, E, distinct=False)
    _check_invariants(idx2, po, G, E, dedup, oracle.layout(idx2, po, G, E, dedup))


def _lexsort_exp_row(idx, po):
    M, topk = idx.shape
    t = np.repeat(np.arange(M), topk)
    k = np.tile(np.arange(topk), M)
    e = idx.ravel()
    p = po[e]
    order = np.lexsort((k, t, e, p))       # last key is primary
    row = np.empty(M * topk, np.int64)
    row[order] = np.arange(M * topk)
    return row.reshape(M, topk)


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_layout_workloads_vs_lexsort(name):
    w = W.get(name)
    idx, po = W.make_routing(w), W.make_placement(w)
    o = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    np.testing.assert_array_equal(o["exp_row"], _lexsort_exp_row(idx, po))
    if w.M <= 16384:
        _check_invariants(idx, po, w.G, w.E_part, w.dedup, o)
    if w.dedup:
        # (p, t) order of the distinct pairs by a numpy unique
        pairs = np.unique(np.stack([po[idx].ravel(), np.repeat(np.arange(w.M), w.topk)], 1), axis=0)
        np.testing.assert_array_equal(o["disp_token"], pairs[:, 1])
        assert o["R_disp"] == pairs.shape[0]


def test_layout_empty_and_degenerate():
    # M = 0
    o = oracle.layout(np.zeros((0, 4), np.int32), np.zeros(8, np.int32), 8, 2, True)
    assert o["R_exp"] == 0 and o["R_disp"] == 0
    assert o["part_offset"].tolist() == [0, 0, 0]
    # every token on one expert
    idx = np.full((50, 1), 3, np.int32)
    po = np.array([0, 0, 1, 1, 2], np.int32)
    o = oracle.layout(idx, po, 5, 3, False)
    assert o["expert_count"].tolist() == [0, 0, 0, 50, 0]
    assert o["expert_offset"].tolist() == [0, 0, 0, 0, 50, 50]
    assert o["exp_row"].ravel().tolist() == list(range(50))
    assert o["part_offset"].tolist() == [0, 0, 50, 50]
