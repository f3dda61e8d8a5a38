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
