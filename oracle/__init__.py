"""CPU oracle of MoE token dispatch / combine (numpy front end).

TEST INFRASTRUCTURE ONLY.  Imported by the tests, by the smoke check and by
the benchmark's CPU-baseline leg, never by the library.  The arithmetic
lives in ``moe_oracle.c`` (plain C, gcc); this module only marshals numpy
arrays.  bf16 data travels as uint16 bit patterns.

Each function follows a passage of the pages:

* :func:`layout` -- Triton-distributed issue #117 test snippet (split counts
  and their cumulative sum), Purlin section 3.1 "Layouts" (scattered-V
  receive buffer), Zyphra news item "correlated expert placement" (dedup: one
  copy of a token per partition);
* :func:`dispatch` -- issue #117 all_to_all_kernel arguments (row copy with
  optional scales, ``WITH_SCALE``), FP8 e4m3 per 128 columns;
* :func:`combine` -- Purlin section 3.3, SCORE (exclusive ownership, ordered
  accumulation);
* :func:`combine_partial` / :func:`combine_reduce` -- the two-level combine
  of a deduplicated dispatch: per (token, partition) reduce in slot order,
  then the token's sum over partitions in partition order;
* :func:`expert_tiles` -- DeepSpeed PR #8180 "Key points": the per-tile
  group map of a grouped GEMM over the expert rows, from the offsets;
* :func:`ep_plan` -- the counts exchange of an expert-parallel all-to-all
  (issue #117 test snippet: split_send_buf -> split_recv_buf,
  send_split_cumsum) into Purlin's transposed-V receive layout (section 3.1:
  destination r holds partition r of every source, in source-rank order).

Pins (tests/test_oracle_*.py, tests/test_golden.py): pure-Python brute force
of the layout definition on every tiny input, layout invariants, the e4m3
encoder against a nearest-value search of the format's decode table and
against torch's float8_e4m3fn cast, bf16 rounding against torch, combine
identities (one-hot / uniform weights) and float64 bounds for both combines,
the tile metadata against a row walk over exp_row, and the dedup ratio of
the hot-pairs batch against the closed form from the pages' statistics.
Every pin set is checked to catch a list of plausible mistakes planted in a
copy of the C source (tests/test_oracle_mutants.py).  Parity of the layout's
row order, the dedup row order and the FP8 conventions (all-zero block,
saturation) rests on stated readings of the pages, not on printed values.
"""
from __future__ import annotations

import ctypes
import os

import numpy as np

from . import build as _build

_lib = None

STATUS_BAD_EXPERT = 1
STATUS_BAD_PART = 2

_i32p = ctypes.POINTER(ctypes.c_int32)


def lib():
    global _lib
    if _lib is None:
        path = _build.build()
        L = ctypes.CDLL(path)
        L.oracle_layout.restype = ctypes.c_int
        L.oracle_layout.argtypes = [ctypes.c_int32] * 5 + [ctypes.c_void_p] * 11
        L.oracle_bf16_round.restype = None
        L.oracle_bf16_round.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_e4m3_encode.restype = None
        L.oracle_e4m3_encode.argtypes = [ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_dispatch.restype = None
        L.oracle_dispatch.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                      ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_combine.restype = ctypes.c_int
        L.oracle_combine.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p,
                                     ctypes.c_void_p, ctypes.c_void_p]
        L.oracle_combine_partial.restype = ctypes.c_int
        L.oracle_combine_partial.argtypes = [ctypes.c_int32] * 4 + [ctypes.c_int64] + [ctypes.c_void_p] * 8
        L.oracle_expert_tiles.restype = ctypes.c_int64
        L.oracle_expert_tiles.argtypes = [ctypes.c_int32, ctypes.c_int32] + [ctypes.c_void_p] * 6
        L.oracle_ep_plan.restype = None
        L.oracle_ep_plan.argtypes = [ctypes.c_int32] * 3 + [ctypes.c_void_p] * 10
        L.oracle_combine_reduce.restype = ctypes.c_int
        L.oracle_combine_reduce.argtypes = [ctypes.c_int32, ctypes.c_int32, ctypes.c_int64] + [ctypes.c_void_p] * 4
        _lib = L
    return _lib


def _p(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def layout(topk_idx, part_of, G: int, E_part: int, dedup: bool) -> dict:
    """Routing layout of ``topk_idx`` [M, topk] under placement ``part_of`` [G].

    Returns int32 arrays: expert_count [G], expert_offset [G+1],
    part_count [E_part], part_offset [E_part+1], exp_row [M, topk],
    disp_token [R_disp], and with dedup disp_row [M, E_part] and
    exp_to_disp [R_exp]; plus the status word and the totals R_exp / R_disp.
    """
    idx = _c(topk_idx, np.int32)
    M, topk = idx.shape
    po = _c(part_of, np.int32)
    assert po.shape == (G,)
    cap = max(M * topk, 1)
    out = dict(
        expert_count=np.zeros(G, np.int32), expert_offset=np.zeros(G + 1, np.int32),
        part_count=np.zeros(E_part, np.int32), part_offset=np.zeros(E_part + 1, np.int32),
        exp_row=np.zeros((M, topk), np.int32), disp_token=np.full(cap, -7, np.int32),
    )
    disp_row = np.zeros((M, E_part), np.int32) if dedup else None
    exp_to_disp = np.full(cap, -7, np.int32) if dedup else None
    st = np.zeros(1, np.int32)
    rc = lib().oracle_layout(M, G, topk, E_part, int(bool(dedup)), _p(idx), _p(po),
                             _p(out["expert_count"]), _p(out["expert_offset"]),
                             _p(out["part_count"]), _p(out["part_offset"]),
                             _p(out["exp_row"]), _p(out["disp_token"]),
                             _p(disp_row), _p(exp_to_disp), _p(st))
    if rc != 0:
        raise MemoryError("oracle_layout: host allocation failed")
    R_exp = int(out["expert_offset"][G])
    R_disp = int(out["part_offset"][E_part])
    out["disp_token"] = out["disp_token"][:R_disp].copy()
    if dedup:
        out["disp_row"] = disp_row
        out["exp_to_disp"] = exp_to_disp[:R_exp].copy()
    out["status"] = int(st[0])
    out["R_exp"] = R_exp
    out["R_disp"] = R_disp
    return out


def dispatch(x_bits, disp_token, fp8: bool, rows=None):
    """Dispatch rows (all, or the listed ``rows``) of token rows ``x_bits``.

    x_bits: uint16 [M, N] bf16 bits.  Returns recv (uint16 or uint8
    [n_rows, N]) and, with fp8, recv_scale float32 [n_rows, N/128].
    """
    x = _c(x_bits, np.uint16)
    N = x.shape[1]
    dt = _c(disp_token, np.int32)
    if rows is None:
        n_rows = dt.shape[0]
        rws = None
    else:
        rws = _c(rows, np.int64)
        n_rows = rws.shape[0]
    if fp8:
        if N % 128:
            raise ValueError("fp8 dispatch needs N % 128 == 0")
        recv = np.zeros((n_rows, N), np.uint8)
        scale = np.zeros((n_rows, N // 128), np.float32)
    else:
        recv = np.zeros((n_rows, N), np.uint16)
        scale = None
    lib().oracle_dispatch(N, int(bool(fp8)), n_rows, _p(rws), _p(dt), _p(x), _p(recv), _p(scale))
    return (recv, scale) if fp8 else recv


def combine(y_bits, topk_weights, exp_row, tokens=None):
    """Gate-weighted combine; returns uint16 bf16 bits [n_tok, N]."""
    y = _c(y_bits, np.uint16)
    N = y.shape[1]
    w = _c(topk_weights, np.float32)
    er = _c(exp_row, np.int32)
    M, topk = er.shape
    if tokens is None:
        n_tok, tk = M, None
    else:
        tk = _c(tokens, np.int64)
        n_tok = tk.shape[0]
    out = np.zeros((n_tok, N), np.uint16)
    rc = lib().oracle_combine(N, topk, n_tok, _p(tk), _p(y), _p(w), _p(er), _p(out))
    if rc != 0:
        raise MemoryError("oracle_combine: host allocation failed")
    return out


def combine_partial(y_bits, topk_weights, topk_idx, part_of, lay, tokens=None):
    """Partition-side reduce of the two-level (dedup) combine: bf16 bits
    [R_disp, N] in dispatch-row space (rows of tokens not listed stay 0)."""
    y = _c(y_bits, np.uint16)
    N = y.shape[1]
    w = _c(topk_weights, np.float32)
    idx = _c(topk_idx, np.int32)
    M, topk = idx.shape
    po = _c(part_of, np.int32)
    er = _c(lay["exp_row"], np.int32)
    dr = _c(lay["disp_row"], np.int32)
    E = dr.shape[1]
    z = np.zeros((max(lay["R_disp"], 1), N), np.uint16)
    if tokens is None:
        n_tok, tk = M, None
    else:
        tk = _c(tokens, np.int64)
        n_tok = tk.shape[0]
    rc = lib().oracle_combine_partial(N, topk, E, po.shape[0], n_tok, _p(tk), _p(idx), _p(po),
                                      _p(y), _p(w), _p(er), _p(dr), _p(z))
    if rc != 0:
        raise MemoryError("oracle_combine_partial: host allocation failed")
    return z[:lay["R_disp"]]


def combine_reduce(z_bits, disp_row, tokens=None):
    """Token-side sum of the two-level combine over partitions (p order)."""
    z = _c(z_bits, np.uint16)
    N = z.shape[1]
    dr = _c(disp_row, np.int32)
    M, E = dr.shape
    if tokens is None:
        n_tok, tk = M, None
    else:
        tk = _c(tokens, np.int64)
        n_tok = tk.shape[0]
    out = np.zeros((n_tok, N), np.uint16)
    rc = lib().oracle_combine_reduce(N, E, n_tok, _p(tk), _p(z), _p(dr), _p(out))
    if rc != 0:
        raise MemoryError("oracle_combine_reduce: host allocation failed")
    return out


def expert_tiles(expert_count, expert_offset, block_m: int) -> dict:
    """Grouped-GEMM tile metadata of a layout: tile_first [G+1] (per expert,
    in row order; [G] = number of tiles) and, per tile, tile_expert,
    tile_row (first row) and tile_rows."""
    cnt = _c(expert_count, np.int32)
    off = _c(expert_offset, np.int32)
    G = cnt.shape[0]
    if block_m < 1:
        raise ValueError("block_m must be >= 1")
    cap = int(sum((int(c) + block_m - 1) // block_m for c in cnt))
    first = np.zeros(G + 1, np.int32)
    te, tr, tn = (np.zeros(max(cap, 1), np.int32) for _ in range(3))
    n = lib().oracle_expert_tiles(G, block_m, _p(cnt), _p(off), _p(first), _p(te), _p(tr), _p(tn))
    assert n == cap
    return dict(tile_first=first, tile_expert=te[:n], tile_row=tr[:n], tile_rows=tn[:n], n_tiles=n)


def ep_plan(part_counts, rank: int, expert_counts=None, part_of=None) -> dict:
    """Exchange plan of ``rank`` among W ranks from every rank's per-partition
    row counts ``part_counts`` [W, W] (row s: rank s's part_count) and,
    optionally, every rank's expert counts ``expert_counts`` [W, G] with the
    placement ``part_of`` [G] (expert -> rank).  Returns int32 arrays
    send_offset [W], src_offset [W], recv_count [W], recv_offset [W+1], and
    with expert counts recv_expert_count [G] and recv_block_offset [W, G];
    plus the status word (8: counts negative, too large or inconsistent)."""
    P = _c(part_counts, np.int32)
    W = P.shape[0]
    assert P.shape == (W, W) and 0 <= rank < W
    out = dict(send_offset=np.zeros(W, np.int32), src_offset=np.zeros(W, np.int32),
               recv_count=np.zeros(W, np.int32), recv_offset=np.zeros(W + 1, np.int32))
    X = po = rec = blk = None
    G = 0
    if expert_counts is not None:
        X = _c(expert_counts, np.int32)
        G = X.shape[1]
        assert X.shape == (W, G)
        po = _c(part_of, np.int32)
        assert po.shape == (G,)
        rec = np.zeros(G, np.int32)
        blk = np.zeros((W, G), np.int32)
    st = np.zeros(1, np.int32)
    lib().oracle_ep_plan(W, rank, G, _p(P), _p(X), _p(po), _p(out["send_offset"]),
                         _p(out["src_offset"]), _p(out["recv_count"]), _p(out["recv_offset"]),
                         _p(rec), _p(blk), _p(st))
    if X is not None:
        out["recv_expert_count"] = rec
        out["recv_block_offset"] = blk
    out["status"] = int(st[0])
    return out


def bf16_round(values) -> np.ndarray:
    """float32 -> bf16 bits (uint16), nearest-even."""
    v = _c(values, np.float32).ravel()
    out = np.zeros(v.shape, np.uint16)
    lib().oracle_bf16_round(v.size, _p(v), _p(out))
    return out.reshape(np.shape(values))


def e4m3_encode(values) -> np.ndarray:
    """float32 -> e4m3 bytes (nearest-even, saturating)."""
    v = _c(values, np.float32).ravel()
    out = np.zeros(v.shape, np.uint8)
    lib().oracle_e4m3_encode(v.size, _p(v), _p(out))
    return out.reshape(np.shape(values))


def step(topk_idx, part_of, topk_weights, x_bits, y_bits, G, E_part, dedup, fp8):
    """Whole path: layout, dispatch of every row, combine of every token."""
    lay = layout(topk_idx, part_of, G, E_part, dedup)
    d = dispatch(x_bits, lay["disp_token"], fp8)
    out = combine(y_bits, topk_weights, lay["exp_row"])
    return lay, d, out


def bf16_bits(t) -> np.ndarray:
    """torch bf16 tensor -> numpy uint16 bit patterns (CPU copy)."""
    import torch
    return t.detach().to("cpu").contiguous().view(torch.int16).numpy().view(np.uint16)


def bits_to_f32(b) -> np.ndarray:
    """bf16 bit patterns -> float32 values (exact)."""
    return (np.asarray(b, np.uint32) << 16).view(np.float32)


__all__ = ["layout", "dispatch", "combine", "combine_partial", "combine_reduce",
           "expert_tiles", "ep_plan", "bf16_round", "e4m3_encode", "step",
           "bf16_bits", "bits_to_f32", "STATUS_BAD_EXPERT", "STATUS_BAD_PART",
           "lib"]

if os.environ.get("MOE_ORACLE_EAGER_BUILD"):
    lib()
