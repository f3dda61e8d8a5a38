"""Fixtures from the pages (tests/golden/, each file citing its source),
checked against the seeded inputs and the oracle (CPU only).

* issue #117's benchmark configuration fixes N, G and topk of the decode,
  M4096, M8192 and prefill workloads and the M values of the latency sweep;
* the Zyphra item's hot-pair statistics fix the hot-pairs workload (128
  experts, 64 hot pairs = a perfect matching, 42% of tokens) and, with its
  placement of 8 hot pairs per partition, the expected dedup ratio in closed
  form: a token saves one of its two copies when both experts share a
  partition, which happens for every hot-pair token and for a uniform pair
  of distinct experts with probability (experts/E - 1) / (experts - 1); the
  oracle's R_disp / R_exp on the seeded batch must match 1 - f/2 within four
  standard deviations of the token sampling.
"""
import math
import os

import numpy as np

import bench
import oracle
import workloads as W

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")


def _fixture(name):
    out = {}
    with open(os.path.join(GOLDEN, name)) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            key, *vals = line.split()
            out[key] = vals
    return out


def test_issue117_benchmark_shapes():
    fx = _fixture("issue117_benchmark.txt")
    N, G, topk = int(fx["N"][0]), int(fx["G"][0]), int(fx["topk"][0])
    for name in ("decode-M128-uniform", "M4096-zipf1.1", "M8192-uniform-fp8",
                 "prefill-M65536-mix-dedup-fp8"):
        w = W.get(name)
        assert (w.N, w.G, w.topk) == (N, G, topk), name
    assert tuple(int(m) for m in fx["M"]) == bench.SWEEP_M
    assert W.get("decode-M128-uniform").M in bench.SWEEP_M


def test_zyphra_hot_pairs_closed_forms():
    fx = _fixture("zyphra_hot_pairs.txt")
    experts, possible = int(fx["experts"][0]), int(fx["pairs_possible"][0])
    hot, h = int(fx["hot_pairs"][0]), float(fx["hot_token_fraction"][0])
    assert math.comb(experts, 2) == possible
    w = W.get("M16384-hotpairs-dedup")
    assert (w.G, w.topk, w.G // 2, w.hot_frac) == (experts, 2, hot, h)
    idx, po = W.make_routing(w), W.make_placement(w)
    # the hot pairs form a perfect matching, packed 8 per partition
    assert np.all(np.bincount(po, minlength=w.E_part) == experts // w.E_part)
    lay = oracle.layout(idx, po, w.G, w.E_part, True)
    assert lay["R_exp"] == w.M * 2
    same = (experts // w.E_part - 1) / (experts - 1)
    f = h + (1 - h) * same
    expected = 1 - f / 2
    got = lay["R_disp"] / lay["R_exp"]
    sigma = math.sqrt(f * (1 - f) / w.M) / 2
    assert abs(got - expected) <= 4 * sigma, (got, expected, sigma)
    # a dedup bound the pages' "up to 58% fewer copies" cannot reach at topk 2
    assert 1 - got < 0.5
