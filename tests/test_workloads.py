"""The seeded input generators: shapes, determinism and the structure the
pages describe (Zyphra: 64 hot pairs of 8,128 carry 42% of tokens and are
packed onto shared partitions; Zipf-skewed and uniform mock routing)."""
import numpy as np
import pytest

import workloads as W


@pytest.mark.parametrize("name", list(W.WORKLOADS))
def test_shapes_and_determinism(name):
    w = W.get(name)
    idx = W.make_routing(w)
    assert idx.shape == (w.M, w.topk) and idx.dtype == np.int32
    assert idx.min() >= 0 and idx.max() < w.G
    # distinct experts per token
    s = np.sort(idx, axis=1)
    assert np.all(np.diff(s, axis=1) > 0)
    np.testing.assert_array_equal(idx, W.make_routing(w))
    po = W.make_placement(w)
    assert po.shape == (w.G,) and po.min() >= 0 and po.max() < w.E_part
    g = W.make_gates(w)
    assert g.shape == (w.M, w.topk) and g.dtype == np.float32
    np.testing.assert_allclose(g.sum(1), 1.0, rtol=1e-5)
    assert not np.array_equal(idx, W.make_routing(w.replace(seed=1)))


def test_contiguous_placement():
    w = W.get("M4096-zipf1.1")
    po = W.make_placement(w)
    np.testing.assert_array_equal(po, np.arange(256) // 32)


def test_hot_pairs_structure():
    w = W.get("M16384-hotpairs-dedup")
    idx = W.make_routing(w)
    po = W.make_placement(w)
    # each partition holds 16 experts = 8 hot pairs
    assert np.all(np.bincount(po, minlength=8) == 16)
    pairs = {tuple(sorted(p)) for p in idx.tolist()}
    assert len(pairs) > 1000
    from collections import Counter
    c = Counter(tuple(sorted(p)) for p in idx.tolist())
    top64 = sum(v for _, v in c.most_common(64)) / w.M
    # 42% hot by construction plus the cold draws that hit a hot pair (~0.5%)
    assert 0.40 < top64 < 0.45
    # every hot pair sits inside one partition
    for (a, b), _ in c.most_common(64):
        assert po[a] == po[b]


def test_zipf_skew():
    w = W.get("M4096-zipf1.1")
    idx = W.make_routing(w)
    cnt = np.sort(np.bincount(idx.ravel(), minlength=256))[::-1]
    # the top expert can appear at most once per token; heavy head, light tail
    assert cnt[0] > 8 * np.median(cnt)
    assert cnt[0] <= w.M
    u = np.bincount(W.make_routing(W.get("M8192-uniform-fp8")).ravel(), minlength=256)
    assert u.max() < 1.25 * u.mean()


def test_mixture_dedup_estimate():
    w = W.get("prefill-M65536-mix-dedup-fp8")
    idx = W.make_routing(w)
    po = W.make_placement(w)
    distinct = sum(len(set(r)) for r in po[idx].tolist())
    # dedup keeps roughly 0.55..0.75 of the M*topk rows for this mixture
    assert 0.55 * w.M * w.topk < distinct < 0.75 * w.M * w.topk


def test_token_tensors_cpu():
    import torch
    w = W.get("decode-M128-uniform").replace(N=256)
    x = W.make_tokens(w)
    assert x.shape == (128, 256) and x.dtype == torch.bfloat16
    assert torch.equal(x, W.make_tokens(w))
    y = W.make_expert_outputs(w)
    assert y.shape == (128 * 8, 256)
    assert abs(float(x.float().std()) - 1.0) < 0.05
