"""Pins of the oracle's combine (CPU only).

* one-hot gates with identity experts (y row = x of its token) return x bit
  for bit;
* uniform gates 1/topk with y = x return x exactly (topk a power of two);
* against the exact float64 sum: within half a bf16 step plus the fp32
  accumulation bound -- a dropped term, a wrong gate index or sign, or a
  transposed operand fails by a whole term;
* gates of pairs the layout left out (exp_row = -1) contribute nothing.
"""
import numpy as np
import pytest

import oracle


def _setup(rng, M, N, G, E, topk, dedup=False):
    idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk].astype(np.int32)
    po = rng.integers(0, E, size=G).astype(np.int32)
    lay = oracle.layout(idx, po, G, E, dedup)
    xb = oracle.bf16_round(rng.standard_normal((M, N)).astype(np.float32))
    return idx, po, lay, xb


def _identity_y(lay, xb, M, topk):
    y = np.zeros((M * topk, xb.shape[1]), np.uint16)
    for t in range(M):
        for k in range(topk):
            y[lay["exp_row"][t, k]] = xb[t]
    return y


@pytest.mark.parametrize("topk", [1, 2, 3, 8])
def test_combine_one_hot_identity(topk):
    rng = np.random.default_rng(topk)
    M, N, G, E = 29, 96, 16, 4
    _, _, lay, xb = _setup(rng, M, N, G, E, topk)
    y = _identity_y(lay, xb, M, topk)
    # pollute the other experts' rows: one-hot gates must ignore them
    w = np.zeros((M, topk), np.float32)
    hot = rng.integers(0, topk, size=M)
    w[np.arange(M), hot] = 1.0
    for t in range(M):
        for k in range(topk):
            if k != hot[t]:
                y[lay["exp_row"][t, k]] = oracle.bf16_round(rng.standard_normal(N).astype(np.float32) * 50)
    out = oracle.combine(y, w, lay["exp_row"])
    np.testing.assert_array_equal(out, xb)


@pytest.mark.parametrize("topk", [1, 2, 4, 8])
def test_combine_uniform_gates_identity(topk):
    rng = np.random.default_rng(100 + topk)
    M, N, G, E = 31, 128, 32, 8
    _, _, lay, xb = _setup(rng, M, N, G, E, topk)
    y = _identity_y(lay, xb, M, topk)
    w = np.full((M, topk), 1.0 / topk, np.float32)
    np.testing.assert_array_equal(oracle.combine(y, w, lay["exp_row"]), xb)


@pytest.mark.parametrize("topk", [2, 5, 8])
def test_combine_within_fp64_bound(topk):
    rng = np.random.default_rng(200 + topk)
    M, N, G, E = 64, 256, 40, 8
    _, _, lay, _ = _setup(rng, M, N, G, E, topk)
    R = M * topk
    y = oracle.bf16_round(rng.standard_normal((R, N)).astype(np.float32))
    z = rng.standard_normal((M, topk))
    w = (np.exp(z) / np.exp(z).sum(1, keepdims=True)).astype(np.float32)
    w[::7, 0] *= -1                          # some negative gates
    out = oracle.bits_to_f32(oracle.combine(y, w, lay["exp_row"])).astype(np.float64)
    yf = oracle.bits_to_f32(y).astype(np.float64)
    terms = w.astype(np.float64)[:, :, None] * yf[lay["exp_row"]]      # [M, topk, N]
    exact = terms.sum(1)
    mag = np.abs(terms).sum(1)
    bound = np.abs(exact) * 2.0 ** -8 + topk * 2.0 ** -23 * mag + 1e-38
    assert np.all(np.abs(out - exact) <= bound)
    # and the bound is tight enough to see one dropped term
    dropped = exact - terms[:, topk - 1, :]
    assert np.mean(np.abs(out - dropped) > bound) > 0.9


def test_combine_skips_left_out_pairs():
    rng = np.random.default_rng(9)
    M, N, G, E, topk = 12, 64, 6, 2, 2
    idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk].astype(np.int32)
    idx[3, 1] = G                           # invalid expert id
    po = rng.integers(0, E, size=G).astype(np.int32)
    lay = oracle.layout(idx, po, G, E, False)
    assert lay["status"] == oracle.STATUS_BAD_EXPERT and lay["exp_row"][3, 1] == -1
    y = oracle.bf16_round(rng.standard_normal((M * topk, N)).astype(np.float32))
    w = np.ones((M, topk), np.float32)
    out = oracle.combine(y, w, lay["exp_row"])
    np.testing.assert_array_equal(out[3], y[lay["exp_row"][3, 0]])


def test_combine_token_subset_matches_full():
    rng = np.random.default_rng(10)
    M, N, G, E, topk = 50, 64, 20, 4, 4
    _, _, lay, _ = _setup(rng, M, N, G, E, topk)
    y = oracle.bf16_round(rng.standard_normal((M * topk, N)).astype(np.float32))
    w = rng.random((M, topk)).astype(np.float32)
    full = oracle.combine(y, w, lay["exp_row"])
    tok = np.array([49, 0, 17], np.int64)
    np.testing.assert_array_equal(oracle.combine(y, w, lay["exp_row"], tokens=tok), full[tok])


# ---------------------------------------------------------------------------
# two-level combine of a deduplicated dispatch
# ---------------------------------------------------------------------------
def _dedup_setup(rng, M, N, G, E, topk, po=None):
    idx = np.argsort(rng.random((M, G)), axis=1)[:, :topk].astype(np.int32)
    if po is None:
        po = rng.integers(0, E, size=G).astype(np.int32)
    lay = oracle.layout(idx, po, G, E, True)
    return idx, po, lay


def _two_level(y, w, idx, po, lay):
    z = oracle.combine_partial(y, w, idx, po, lay)
    return z, oracle.combine_reduce(z, lay["disp_row"])


@pytest.mark.parametrize("topk", [1, 2, 4, 8])
def test_two_level_one_hot_identity(topk):
    rng = np.random.default_rng(300 + topk)
    M, N, G, E = 40, 64, 16, 4
    idx, po, lay = _dedup_setup(rng, M, N, G, E, topk)
    xb = oracle.bf16_round(rng.standard_normal((M, N)).astype(np.float32))
    y = oracle.bf16_round(rng.standard_normal((M * topk, N)).astype(np.float32) * 30)
    hot = rng.integers(0, topk, size=M)
    w = np.zeros((M, topk), np.float32)
    w[np.arange(M), hot] = 1.0
    for t in range(M):
        y[lay["exp_row"][t, hot[t]]] = xb[t]
    z, out = _two_level(y, w, idx, po, lay)
    np.testing.assert_array_equal(out, xb)
    # the partition of the hot slot carries x, every other partition +0
    for t in range(M):
        for p in range(E):
            r = lay["disp_row"][t, p]
            if r < 0:
                continue
            want = xb[t] if po[idx[t, hot[t]]] == p else np.zeros(N, np.uint16)
            np.testing.assert_array_equal(z[r], want)


@pytest.mark.parametrize("topk", [2, 4, 8])
def test_two_level_colocated_uniform_identity(topk):
    """All of a token's experts in one partition: the partition sum of
    x/topk terms is x exactly, the token sum over one partition is x."""
    rng = np.random.default_rng(400 + topk)
    M, N, E = 30, 64, 4
    G = E * topk
    po = (np.arange(G) // topk).astype(np.int32)
    grp = rng.integers(0, E, size=M)
    idx = np.stack([rng.permutation(topk) + grp[t] * topk for t in range(M)]).astype(np.int32)
    lay = oracle.layout(idx, po, G, E, True)
    assert lay["R_disp"] == M
    xb = oracle.bf16_round(rng.standard_normal((M, N)).astype(np.float32))
    y = np.zeros((M * topk, N), np.uint16)
    for t in range(M):
        for k in range(topk):
            y[lay["exp_row"][t, k]] = xb[t]
    w = np.full((M, topk), 1.0 / topk, np.float32)
    z, out = _two_level(y, w, idx, po, lay)
    np.testing.assert_array_equal(out, xb)
    np.testing.assert_array_equal(z, xb[lay["disp_token"]])


@pytest.mark.parametrize("topk,E", [(2, 8), (5, 3), (8, 8), (8, 2)])
def test_two_level_within_fp64_bounds(topk, E):
    rng = np.random.default_rng(500 + topk * 10 + E)
    M, N, G = 48, 128, 32
    idx, po, lay = _dedup_setup(rng, M, N, G, E, topk)
    y = oracle.bf16_round(rng.standard_normal((M * topk, N)).astype(np.float32))
    z0 = rng.standard_normal((M, topk))
    w = (np.exp(z0) / np.exp(z0).sum(1, keepdims=True)).astype(np.float32)
    w[::5, 0] *= -1
    z, out = _two_level(y, w, idx, po, lay)
    yf = oracle.bits_to_f32(y).astype(np.float64)
    zf = oracle.bits_to_f32(z).astype(np.float64)
    outf = oracle.bits_to_f32(out).astype(np.float64)
    terms = w.astype(np.float64)[:, :, None] * yf[lay["exp_row"]]     # [M, topk, N]
    exact = terms.sum(1)
    mag_all = np.abs(terms).sum(1)
    part_mag = np.zeros((M, N))
    for t in range(M):
        for p in range(E):
            r = lay["disp_row"][t, p]
            if r < 0:
                continue
            sel = po[idx[t]] == p
            ex_p = terms[t, sel].sum(0)
            mag_p = np.abs(terms[t, sel]).sum(0)
            # each partition row: one bf16 rounding of its own slots' sum
            assert np.all(np.abs(zf[r] - ex_p) <= np.abs(ex_p) * 2.0 ** -8 + topk * 2.0 ** -23 * mag_p + 1e-38)
            part_mag += np.abs(ex_p) + mag_p * 2.0 ** -20
    bound = np.abs(exact) * 2.0 ** -8 + part_mag * 2.0 ** -7 + E * 2.0 ** -23 * mag_all + 1e-37
    assert np.all(np.abs(outf - exact) <= bound)
