"""Pins of the oracle's grouped-GEMM tile metadata (CPU only).

The reference construction here walks the expert rows one by one, using the
row -> expert map that the layout's exp_row gives (not the counts or offsets
the oracle reads), and opens a new tile whenever the expert changes or the
tile is full.  On top of that:

* block_m = 1 gives one tile per row, labelled with the row's expert;
* block_m >= every count gives one tile per non-empty expert, at its offset;
* for any block_m the tiles cover [0, R_exp) once, in row order, never
  straddle two experts, and expert e has ceil(count / block_m) of them;
* tile_first of an expert is the number of tiles that start before its
  first row (also for empty experts and experts placed nowhere).
"""
import numpy as np
import pytest

import oracle


def _layout(rng, M, G, E, topk, dedup=False, po=None, idx=None):
    if idx is None:
        idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk].astype(np.int32)
    if po is None:
        po = rng.integers(0, E, size=G).astype(np.int32)
    return idx, po, oracle.layout(idx, po, G, E, dedup)


def _row_expert(idx, lay):
    """Expert of every expert row, from exp_row alone."""
    R = int(lay["R_exp"])
    owner = np.full(R, -1, np.int64)
    er = lay["exp_row"]
    for t in range(idx.shape[0]):
        for k in range(idx.shape[1]):
            if er[t, k] >= 0:
                owner[er[t, k]] = idx[t, k]
    assert np.all(owner >= 0)
    return owner


def _walk(owner, block_m):
    """Tiles by walking the rows: a new tile at each change of expert or when full."""
    te, tr, tn = [], [], []
    for r, e in enumerate(owner):
        if not te or te[-1] != e or tn[-1] == block_m:
            te.append(int(e))
            tr.append(r)
            tn.append(0)
        tn[-1] += 1
    return np.array(te, np.int64), np.array(tr, np.int64), np.array(tn, np.int64)


CASES = [
    (64, 16, 4, 2, False, "random"),
    (200, 40, 8, 5, True, "random"),
    (97, 256, 8, 8, False, "contiguous"),
    (50, 12, 3, 4, False, "some-unplaced"),
    (1, 8, 2, 1, False, "random"),
    (0, 8, 2, 2, False, "random"),
]


@pytest.mark.parametrize("M,G,E,topk,dedup,placement", CASES)
@pytest.mark.parametrize("block_m", [1, 3, 16, 128, 1 << 20])
def test_tiles_match_the_row_walk(M, G, E, topk, dedup, placement, block_m):
    rng = np.random.default_rng(M * 7 + G + block_m % 97)
    po = None
    if placement == "contiguous":
        po = (np.arange(G) * E // G).astype(np.int32)
    elif placement == "some-unplaced":
        po = rng.integers(0, E, size=G).astype(np.int32)
        po[[1, 5]] = E                               # placed nowhere: zero rows
    idx, po, lay = _layout(rng, M, G, E, topk, dedup, po)
    owner = _row_expert(idx, lay) if M else np.zeros(0, np.int64)
    te, tr, tn = _walk(owner, block_m)
    got = oracle.expert_tiles(lay["expert_count"], lay["expert_offset"], block_m)
    assert got["n_tiles"] == len(te)
    np.testing.assert_array_equal(got["tile_expert"], te)
    np.testing.assert_array_equal(got["tile_row"], tr)
    np.testing.assert_array_equal(got["tile_rows"], tn)
    # first tile of each expert: the tiles that start before its first row
    for e in range(G):
        assert got["tile_first"][e] == int(np.sum(tr < lay["expert_offset"][e]))
    assert got["tile_first"][G] == len(te)


def test_block_of_one_row_labels_every_row():
    rng = np.random.default_rng(1)
    idx, po, lay = _layout(rng, 120, 32, 4, 6)
    got = oracle.expert_tiles(lay["expert_count"], lay["expert_offset"], 1)
    np.testing.assert_array_equal(got["tile_row"], np.arange(lay["R_exp"]))
    np.testing.assert_array_equal(got["tile_expert"], _row_expert(idx, lay))
    assert np.all(got["tile_rows"] == 1)


def test_one_tile_per_expert_when_block_is_large():
    rng = np.random.default_rng(2)
    idx, po, lay = _layout(rng, 300, 24, 6, 4)
    cnt, off = lay["expert_count"], lay["expert_offset"]
    got = oracle.expert_tiles(cnt, off, int(cnt.max()))
    nz = np.nonzero(cnt)[0]
    order = nz[np.argsort(off[nz])]
    np.testing.assert_array_equal(got["tile_expert"], order)
    np.testing.assert_array_equal(got["tile_row"], off[order])
    np.testing.assert_array_equal(got["tile_rows"], cnt[order])


@pytest.mark.parametrize("block_m", [2, 7, 64])
def test_cover_once_and_ceil_count(block_m):
    rng = np.random.default_rng(3 + block_m)
    idx, po, lay = _layout(rng, 500, 64, 8, 8, dedup=True)
    cnt, off = lay["expert_count"], lay["expert_offset"]
    got = oracle.expert_tiles(cnt, off, block_m)
    tr, tn, te = got["tile_row"], got["tile_rows"], got["tile_expert"]
    assert tr[0] == 0 and np.all(tr[1:] == tr[:-1] + tn[:-1]) and tr[-1] + tn[-1] == lay["R_exp"]
    assert np.all((tn >= 1) & (tn <= block_m))
    assert np.all(tr >= off[te]) and np.all(tr + tn <= off[te] + cnt[te])
    np.testing.assert_array_equal(np.bincount(te, minlength=64), -(-cnt // block_m))
    full = np.r_[te[1:] == te[:-1], False]           # every tile but an expert's last is full
    assert np.all(tn[full] == block_m)
