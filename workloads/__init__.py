"""Seeded synthetic inputs for MoE token dispatch / combine.

This module only draws inputs: routing (top-k expert ids), gate weights, the
expert-to-partition placement map, token rows ``x`` and expert outputs ``y``.
It holds none of the path's arithmetic (no layout, no permute, no
quantisation, no reduction), so both the CUDA path and the CPU oracle consume
the same bytes from it without sharing any code with each other.

Workload shapes follow the pages:

* Triton-distributed issue #117, "Benchmark Configuration": hidden N = 7168,
  G = 256 experts, topk = 8, bf16 tokens, M swept from 2 to 512.
* Zyphra news item, "Zyphra finds MoE expert routing has strong, exploitable
  pair patterns": 64 of 8,128 expert pairs (8,128 = C(128, 2), hence G = 128
  at topk = 2) carry 42% of the tokens of one layer; "correlated expert
  placement" puts experts that are chosen together on the same GPU.
* DODOCO abstract ("Diagnosing Overhead in Dispatch Operations"): mock
  routing is usually uniform or Zipf-skewed, so both are generated.

Random draws:

* uniform routing: ``topk`` distinct experts per token, uniformly, in random
  slot order;
* Zipf(s) routing: expert popularity p_r ~ r^-s over ranks r = 1..G, ranks
  mapped to experts through a seeded permutation; ``topk`` draws without
  replacement per token (sequential renormalised draws, done as Gumbel-top-k
  on log p), slot order = draw order;
* hot-pair routing: a seeded perfect matching of the G experts into G/2 hot
  pairs; a fraction ``hot_frac`` of the tokens takes a hot pair drawn
  uniformly (random slot order), the rest a uniform pair of distinct experts;
* mixture routing: per token, uniform with probability ``mix_frac`` else Zipf;
* gates: softmax of N(0, 1) logits over the ``topk`` slots, stored as fp32;
* ``x`` and ``y``: N(0, 1) rounded to bf16, drawn with torch's generator on
  the device that will hold them (Philox on CUDA, the CPU generator on CPU).

Every stream is derived from one root seed with ``numpy.random.SeedSequence``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

__all__ = ["Workload", "WORKLOADS", "get", "make_routing", "make_placement",
           "make_gates", "make_tokens", "make_expert_outputs", "make_inputs"]


@dataclasses.dataclass(frozen=True)
class Workload:
    """Sizes and input recipe of one dispatch/combine problem."""
    name: str
    M: int                 # tokens
    N: int                 # hidden size (bf16 columns)
    G: int                 # experts
    topk: int              # experts per token
    E_part: int            # destination partitions
    routing: str           # "uniform" | "zipf" | "hot_pairs" | "mix"
    placement: str         # "contiguous" | "hot_pairs"
    dedup: bool = False
    fp8: bool = False
    zipf_s: float = 1.1
    hot_frac: float = 0.42
    mix_frac: float = 0.5
    seed: int = 0

    def replace(self, **kw) -> "Workload":
        return dataclasses.replace(self, **kw)


# The five configurations of the hot path, named by what they are.
WORKLOADS = {
    "decode-M128-uniform": Workload(
        "decode-M128-uniform", M=128, N=7168, G=256, topk=8, E_part=8,
        routing="uniform", placement="contiguous"),
    "M4096-zipf1.1": Workload(
        "M4096-zipf1.1", M=4096, N=7168, G=256, topk=8, E_part=8,
        routing="zipf", zipf_s=1.1, placement="contiguous"),
    "M16384-hotpairs-dedup": Workload(
        "M16384-hotpairs-dedup", M=16384, N=4096, G=128, topk=2, E_part=8,
        routing="hot_pairs", hot_frac=0.42, placement="hot_pairs", dedup=True),
    "M8192-uniform-fp8": Workload(
        "M8192-uniform-fp8", M=8192, N=7168, G=256, topk=8, E_part=8,
        routing="uniform", placement="contiguous", fp8=True),
    "prefill-M65536-mix-dedup-fp8": Workload(
        "prefill-M65536-mix-dedup-fp8", M=65536, N=7168, G=256, topk=8,
        E_part=8, routing="mix", zipf_s=1.2, mix_frac=0.5,
        placement="contiguous", dedup=True, fp8=True),
}


def get(name: str) -> Workload:
    return WORKLOADS[name]


# ---------------------------------------------------------------------------
# seed streams
# ---------------------------------------------------------------------------
_STREAMS = ("routing", "gates", "placement", "x", "y", "mix")


def _children(seed: int):
    kids = np.random.SeedSequence(seed).spawn(len(_STREAMS))
    return dict(zip(_STREAMS, kids))


def _rng(seed: int, stream: str) -> np.random.Generator:
    return np.random.default_rng(_children(seed)[stream])


def _torch_seed(seed: int, stream: str) -> int:
    return int(_children(seed)[stream].generate_state(1, np.uint64)[0] & ((1 << 63) - 1))


# ---------------------------------------------------------------------------
# routing
# ---------------------------------------------------------------------------
def _uniform_distinct(rng, M, G, topk):
    keys = rng.random((M, G))
    return np.argsort(keys, axis=1, kind="stable")[:, :topk]


def _zipf_probs(G, s, rng):
    ranks = np.arange(1, G + 1, dtype=np.float64)
    p_rank = ranks ** (-s)
    p_rank /= p_rank.sum()
    perm = rng.permutation(G)           # rank r -> expert perm[r-1]
    p = np.empty(G)
    p[perm] = p_rank
    return p


def _gumbel_topk(rng, logp, M, topk):
    g = rng.gumbel(size=(M, logp.shape[0]))
    keys = logp[None, :] + g
    order = np.argsort(-keys, axis=1, kind="stable")
    return order[:, :topk]


def _hot_pairs(rng, G):
    perm = rng.permutation(G)
    return perm.reshape(G // 2, 2)


def make_routing(w: Workload) -> np.ndarray:
    """topk_idx [M, topk] int32 for workload ``w`` (seeded)."""
    rng = _rng(w.seed, "routing")
    M, G, topk = w.M, w.G, w.topk
    if w.routing == "uniform":
        idx = _uniform_distinct(rng, M, G, topk)
    elif w.routing == "zipf":
        p = _zipf_probs(G, w.zipf_s, rng)
        idx = _gumbel_topk(rng, np.log(p), M, topk)
    elif w.routing == "mix":
        p = _zipf_probs(G, w.zipf_s, rng)
        uni = _uniform_distinct(rng, M, G, topk)
        zpf = _gumbel_topk(rng, np.log(p), M, topk)
        pick = _rng(w.seed, "mix").random(M) < w.mix_frac
        idx = np.where(pick[:, None], uni, zpf)
    elif w.routing == "hot_pairs":
        if topk != 2:
            raise ValueError("hot-pair routing draws pairs: topk must be 2")
        pairs = _hot_pairs(_rng(w.seed, "placement"), G)
        hot = rng.random(M) < w.hot_frac
        which = rng.integers(0, pairs.shape[0], size=M)
        swap = rng.random(M) < 0.5
        hp = pairs[which]
        hp = np.where(swap[:, None], hp[:, ::-1], hp)
        a = rng.integers(0, G, size=M)
        b = rng.integers(0, G - 1, size=M)
        b = b + (b >= a)
        cold = np.stack([a, b], axis=1)
        idx = np.where(hot[:, None], hp, cold)
    else:
        raise ValueError(f"unknown routing {w.routing!r}")
    return np.ascontiguousarray(idx, dtype=np.int32)


def make_placement(w: Workload) -> np.ndarray:
    """part_of [G] int32: the expert -> destination-partition map."""
    G, E = w.G, w.E_part
    if w.placement == "contiguous":
        part = (np.arange(G, dtype=np.int64) * E) // G
    elif w.placement == "hot_pairs":
        pairs = _hot_pairs(_rng(w.seed, "placement"), G)
        n_pairs = pairs.shape[0]
        part = np.empty(G, dtype=np.int64)
        for i in range(n_pairs):           # pairs packed E-way, in pair order
            part[pairs[i]] = (i * E) // n_pairs
    else:
        raise ValueError(f"unknown placement {w.placement!r}")
    return np.ascontiguousarray(part, dtype=np.int32)


def make_gates(w: Workload) -> np.ndarray:
    """topk_weights [M, topk] fp32 = softmax of N(0,1) logits per token."""
    rng = _rng(w.seed, "gates")
    z = rng.standard_normal((w.M, w.topk))
    z = z - z.max(axis=1, keepdims=True)
    e = np.exp(z)
    return np.ascontiguousarray(e / e.sum(axis=1, keepdims=True), dtype=np.float32)


def _randn_bf16(shape, seed, device, chunk_rows: int = 1 << 16):
    import torch
    g = torch.Generator(device=device)
    g.manual_seed(seed)
    out = torch.empty(shape, dtype=torch.bfloat16, device=device)
    rows = shape[0]
    for r0 in range(0, rows, chunk_rows):
        r1 = min(rows, r0 + chunk_rows)
        out[r0:r1] = torch.randn((r1 - r0,) + tuple(shape[1:]), generator=g,
                                 device=device, dtype=torch.float32).to(torch.bfloat16)
    return out


def make_tokens(w: Workload, device="cpu"):
    """x [M, N] bf16 torch tensor, N(0, 1)."""
    return _randn_bf16((w.M, w.N), _torch_seed(w.seed, "x"), device)


def make_expert_outputs(w: Workload, rows: Optional[int] = None, device="cpu"):
    """y [rows, N] bf16 torch tensor, N(0, 1); rows defaults to M*topk."""
    rows = w.M * w.topk if rows is None else rows
    return _randn_bf16((rows, w.N), _torch_seed(w.seed, "y"), device)


def make_inputs(w: Workload, device="cpu", with_y: bool = True) -> dict:
    """All inputs of one problem: numpy routing/gates/placement, torch x/y."""
    d = dict(topk_idx=make_routing(w), topk_weights=make_gates(w),
             part_of=make_placement(w), x=make_tokens(w, device))
    if with_y:
        d["y"] = make_expert_outputs(w, device=device)
    return d
