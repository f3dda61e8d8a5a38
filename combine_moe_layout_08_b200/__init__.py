"""B200 (sm_100a) MoE token dispatch / combine.

Python face of libmoe_layout.so, with the C names:

* :func:`moe_layout`   -- routing layout (counts, prefix sums, row indices)
* :func:`moe_dispatch` -- dispatch permute, optional dedup and FP8 e4m3 cast
* :func:`moe_combine`  -- gate-weighted, slot-ordered combine
* :func:`moe_combine_partial` / :func:`moe_combine_reduce` -- the two-level
  combine of a deduplicated dispatch (per partition, then per token)
* :func:`moe_ep_plan` -- offsets of an expert-parallel exchange over W ranks
  from every rank's counts; :func:`ep_all_gather_counts` gathers those counts
  over a process group (the counts exchange itself, torch.distributed)
* :func:`moe_ep_dispatch` / :func:`moe_ep_combine` /
  :func:`moe_ep_combine_reduce` -- the expert-parallel data plane: rows pushed
  into, and outputs pulled from, every rank's buffers through a table of
  device pointers (:class:`EpPeers`)

Tensors are passed as device pointers with the current CUDA stream; this
module checks dtypes, shapes and devices, allocates nothing inside the calls
and computes nothing itself.  :func:`alloc_layout` and :class:`MoEBuffers`
are conveniences that allocate caller-side buffers at worst-case capacity.
"""
from __future__ import annotations

import ctypes
import dataclasses
from typing import Optional

import torch

from . import _lib
from ._lib import (MOE_MAX_E_PART, MOE_MAX_G, MOE_MAX_N, MOE_MAX_TOPK, MOE_STATIC_SCRATCH_BYTES,
                   MOE_STATUS_BAD_COUNT, MOE_STATUS_BAD_EXPERT,
                   MOE_STATUS_BAD_PART, MOE_STATUS_BAD_ROW, MoEError)

__all__ = ["MoEProblem", "MoELayout", "MoEBuffers", "MoEError", "alloc_layout",
           "layout_workspace_size", "moe_layout", "moe_layout_static", "moe_dispatch",
           "moe_layout_dispatch", "moe_layout_dispatch_fused", "moe_expert_tiles",
           "expert_tiles_capacity", "alloc_expert_tiles", "ExpertTiles", "moe_combine", "moe_combine_partial", "moe_combine_reduce",
           "moe_status_string", "moe_abi_version", "MOE_STATUS_BAD_EXPERT",
           "MOE_STATUS_BAD_PART", "MOE_STATUS_BAD_ROW", "MOE_STATUS_BAD_COUNT", "MOE_MAX_G",
           "MOE_MAX_E_PART", "EpPlan", "alloc_ep_plan", "moe_ep_plan", "ep_all_gather_counts",
           "EpPeers", "ep_peers", "moe_ep_dispatch", "moe_ep_combine", "moe_ep_combine_reduce",
           "MOE_MAX_TOPK", "MOE_MAX_N"]


@dataclasses.dataclass(frozen=True)
class MoEProblem:
    M: int
    N: int
    G: int
    topk: int
    E_part: int
    dedup: bool = False
    fp8: bool = False

    def struct(self) -> _lib.ProblemStruct:
        return _lib.ProblemStruct(self.M, self.N, self.G, self.topk, self.E_part,
                                  int(bool(self.dedup)), int(bool(self.fp8)))

    @property
    def capacity(self) -> int:
        """Receive-buffer rows at worst case (M * topk)."""
        return self.M * self.topk


@dataclasses.dataclass
class MoELayout:
    """Device arrays of one layout (int32), see ``moe_layout_t``."""
    expert_count: torch.Tensor
    expert_offset: torch.Tensor
    part_count: torch.Tensor
    part_offset: torch.Tensor
    exp_row: torch.Tensor
    disp_token: torch.Tensor
    status: torch.Tensor
    disp_row: Optional[torch.Tensor] = None
    exp_to_disp: Optional[torch.Tensor] = None

    def struct(self) -> _lib.LayoutStruct:
        def p(t):
            return None if t is None else t.data_ptr()
        return _lib.LayoutStruct(p(self.expert_count), p(self.expert_offset), p(self.part_count),
                                 p(self.part_offset), p(self.exp_row), p(self.disp_token),
                                 p(self.disp_row), p(self.exp_to_disp), p(self.status))


def moe_abi_version() -> int:
    return _lib.load().moe_abi_version()


def moe_status_string(code: int) -> str:
    return _lib.load().moe_status_string(code).decode()


def layout_workspace_size(prob: MoEProblem) -> int:
    s = prob.struct()
    return int(_lib.load().moe_layout_workspace_size(ctypes.byref(s)))


def alloc_layout(prob: MoEProblem, device="cuda") -> MoELayout:
    """Layout arrays at worst-case capacity on ``device`` (uninitialised)."""
    cap = max(prob.capacity, 1)
    i32 = dict(dtype=torch.int32, device=device)
    return MoELayout(
        expert_count=torch.empty(prob.G, **i32), expert_offset=torch.empty(prob.G + 1, **i32),
        part_count=torch.empty(prob.E_part, **i32), part_offset=torch.empty(prob.E_part + 1, **i32),
        exp_row=torch.empty(cap, **i32), disp_token=torch.empty(cap, **i32),
        status=torch.empty(1, **i32),
        disp_row=torch.empty(max(prob.M * prob.E_part, 1), **i32) if prob.dedup else None,
        exp_to_disp=torch.empty(cap, **i32) if prob.dedup else None)


def _stream(t: torch.Tensor, stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream(t.device)
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _check(t, name, dtype, numel=None, device=None):
    if t is None:
        raise ValueError(f"{name} is required")
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if numel is not None and t.numel() < numel:
        raise ValueError(f"{name}: needs >= {numel} elements, has {t.numel()}")
    if device is not None and t.device != device:
        raise ValueError(f"{name} is on {t.device}, expected {device}")


def _check_layout(prob: MoEProblem, lay: MoELayout, device):
    cap = prob.capacity
    _check(lay.expert_count, "expert_count", torch.int32, prob.G, device)
    _check(lay.expert_offset, "expert_offset", torch.int32, prob.G + 1, device)
    _check(lay.part_count, "part_count", torch.int32, prob.E_part, device)
    _check(lay.part_offset, "part_offset", torch.int32, prob.E_part + 1, device)
    _check(lay.exp_row, "exp_row", torch.int32, cap, device)
    _check(lay.disp_token, "disp_token", torch.int32, cap, device)
    _check(lay.status, "status", torch.int32, 1, device)
    if prob.dedup:
        _check(lay.disp_row, "disp_row", torch.int32, prob.M * prob.E_part, device)
        _check(lay.exp_to_disp, "exp_to_disp", torch.int32, cap, device)


def moe_layout(prob: MoEProblem, topk_idx: torch.Tensor, part_of: torch.Tensor,
               lay: MoELayout, workspace: torch.Tensor, stream=None) -> None:
    """Routing layout of ``topk_idx`` [M, topk] int32 under ``part_of`` [G] int32."""
    dev = part_of.device
    _check(topk_idx, "topk_idx", torch.int32, prob.M * prob.topk, dev)
    _check(part_of, "part_of", torch.int32, prob.G, dev)
    _check(workspace, "workspace", torch.uint8, None, dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_layout(ctypes.byref(s), topk_idx.data_ptr(), part_of.data_ptr(),
                                ctypes.byref(l), workspace.data_ptr(), workspace.numel(),
                                _stream(part_of, stream))
    if rc:
        raise MoEError("moe_layout", rc)


def moe_layout_static(prob: MoEProblem, topk_idx: torch.Tensor, part_of: torch.Tensor,
                      lay: MoELayout, stream=None) -> None:
    """moe_layout without a workspace argument, for callers that cannot
    allocate device memory: the scratch is a fixed device array inside the
    library (MOE_STATIC_SCRATCH_BYTES), shared by every call.  Calls that
    overlap on the GPU race on it; the first call in each CUDA context (the
    first on a device, and the first after its context was re-created) looks
    up the array's address and must come before any stream capture."""
    dev = part_of.device
    _check(topk_idx, "topk_idx", torch.int32, prob.M * prob.topk, dev)
    _check(part_of, "part_of", torch.int32, prob.G, dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_layout_static(ctypes.byref(s), topk_idx.data_ptr(), part_of.data_ptr(),
                                       ctypes.byref(l), _stream(part_of, stream))
    if rc:
        raise MoEError("moe_layout_static", rc)


def moe_dispatch(prob: MoEProblem, x: torch.Tensor, lay: MoELayout, recv_x: torch.Tensor,
                 recv_scale: Optional[torch.Tensor] = None, stream=None) -> None:
    """Dispatch rows of ``x`` [M, N] bf16 into ``recv_x`` (bf16, or uint8 with fp8)."""
    dev = x.device
    cap = prob.capacity
    _check(x, "x", torch.bfloat16, prob.M * prob.N, dev)
    _check(recv_x, "recv_x", torch.uint8 if prob.fp8 else torch.bfloat16, cap * prob.N, dev)
    if prob.fp8:
        _check(recv_scale, "recv_scale", torch.float32, cap * (prob.N // 128), dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_dispatch(ctypes.byref(s), x.data_ptr(), ctypes.byref(l), recv_x.data_ptr(),
                                  recv_scale.data_ptr() if recv_scale is not None else None,
                                  _stream(x, stream))
    if rc:
        raise MoEError("moe_dispatch", rc)


def moe_layout_dispatch(prob: MoEProblem, topk_idx: torch.Tensor, part_of: torch.Tensor,
                        lay: MoELayout, workspace: torch.Tensor, x: torch.Tensor,
                        recv_x: torch.Tensor, recv_scale: Optional[torch.Tensor] = None,
                        tiles: Optional["ExpertTiles"] = None, stream=None) -> None:
    """moe_layout then moe_dispatch in one call (bit-identical results); small
    batches run as one kernel (see ``moe_layout_dispatch_fused``).  ``tiles``
    also fills the grouped-GEMM tile metadata from the same kernels."""
    dev = x.device
    cap = prob.capacity
    _check(topk_idx, "topk_idx", torch.int32, prob.M * prob.topk, dev)
    _check(part_of, "part_of", torch.int32, prob.G, dev)
    _check(workspace, "workspace", torch.uint8, None, dev)
    _check(x, "x", torch.bfloat16, prob.M * prob.N, dev)
    _check(recv_x, "recv_x", torch.uint8 if prob.fp8 else torch.bfloat16, cap * prob.N, dev)
    if prob.fp8:
        _check(recv_scale, "recv_scale", torch.float32, cap * (prob.N // 128), dev)
    _check_layout(prob, lay, dev)
    if tiles is not None:
        _check_tiles(prob, tiles, dev)
    s, l = prob.struct(), lay.struct()
    ts = tiles.struct() if tiles is not None else None
    rc = _lib.load().moe_layout_dispatch(
        ctypes.byref(s), topk_idx.data_ptr(), part_of.data_ptr(), ctypes.byref(l),
        workspace.data_ptr(), workspace.numel(), x.data_ptr(), recv_x.data_ptr(),
        recv_scale.data_ptr() if recv_scale is not None else None,
        ctypes.byref(ts) if ts is not None else None, _stream(x, stream))
    if rc:
        raise MoEError("moe_layout_dispatch", rc)


def moe_layout_dispatch_fused(prob: MoEProblem) -> bool:
    """True if moe_layout_dispatch runs ``prob`` as one kernel."""
    s = prob.struct()
    return bool(_lib.load().moe_layout_dispatch_fused(ctypes.byref(s)))


def expert_tiles_capacity(prob: MoEProblem, block_m: int) -> int:
    """Entries each tile array of moe_expert_tiles needs (0: invalid)."""
    s = prob.struct()
    return int(_lib.load().moe_expert_tiles_capacity(ctypes.byref(s), block_m))


@dataclasses.dataclass
class ExpertTiles:
    """Grouped-GEMM tile metadata on the device (see moe_expert_tiles)."""
    block_m: int
    tile_first: torch.Tensor   # [G+1] int32
    tile_expert: torch.Tensor  # [cap] int32
    tile_row: torch.Tensor     # [cap] int32
    tile_rows: torch.Tensor    # [cap] int32

    def struct(self) -> _lib.TilesStruct:
        return _lib.TilesStruct(self.block_m, self.tile_first.data_ptr(),
                                self.tile_expert.data_ptr(), self.tile_row.data_ptr(),
                                self.tile_rows.data_ptr())


def _check_tiles(prob: MoEProblem, tiles: ExpertTiles, device):
    cap = expert_tiles_capacity(prob, tiles.block_m)
    if cap == 0:
        raise ValueError(f"invalid block_m={tiles.block_m}")
    _check(tiles.tile_first, "tile_first", torch.int32, prob.G + 1, device)
    for name in ("tile_expert", "tile_row", "tile_rows"):
        _check(getattr(tiles, name), name, torch.int32, cap, device)


def alloc_expert_tiles(prob: MoEProblem, block_m: int, device) -> ExpertTiles:
    cap = expert_tiles_capacity(prob, block_m)
    if cap == 0:
        raise ValueError(f"invalid problem or block_m={block_m}")
    i32 = dict(dtype=torch.int32, device=device)
    return ExpertTiles(block_m, torch.empty(prob.G + 1, **i32), torch.empty(cap, **i32),
                       torch.empty(cap, **i32), torch.empty(cap, **i32))


def moe_expert_tiles(prob: MoEProblem, part_of: torch.Tensor, lay: MoELayout,
                     tiles: ExpertTiles, stream=None) -> None:
    """Per-tile expert map of a grouped GEMM over the layout's expert rows,
    tiles of ``tiles.block_m`` rows in row order (after moe_layout)."""
    dev = part_of.device
    _check(part_of, "part_of", torch.int32, prob.G, dev)
    _check_tiles(prob, tiles, dev)
    _check_layout(prob, lay, dev)
    s, l, ts = prob.struct(), lay.struct(), tiles.struct()
    rc = _lib.load().moe_expert_tiles(ctypes.byref(s), part_of.data_ptr(), ctypes.byref(l),
                                      ctypes.byref(ts), _stream(part_of, stream))
    if rc:
        raise MoEError("moe_expert_tiles", rc)


def moe_combine(prob: MoEProblem, y: torch.Tensor, topk_weights: torch.Tensor, lay: MoELayout,
                out: torch.Tensor, stream=None) -> None:
    """out [M, N] bf16 = gate-weighted sum of the expert rows ``y`` [M*topk, N] bf16."""
    dev = y.device
    _check(y, "y", torch.bfloat16, prob.capacity * prob.N, dev)
    _check(topk_weights, "topk_weights", torch.float32, prob.M * prob.topk, dev)
    _check(out, "out", torch.bfloat16, prob.M * prob.N, dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_combine(ctypes.byref(s), y.data_ptr(), topk_weights.data_ptr(),
                                 ctypes.byref(l), out.data_ptr(), _stream(y, stream))
    if rc:
        raise MoEError("moe_combine", rc)


def moe_combine_partial(prob: MoEProblem, y: torch.Tensor, topk_weights: torch.Tensor,
                        lay: MoELayout, z: torch.Tensor, stream=None) -> None:
    """Partition side of the two-level (dedup) combine: z [M*topk, N] bf16 in
    dispatch-row space, one row per (token, partition)."""
    dev = y.device
    if not prob.dedup:
        raise ValueError("the two-level combine needs a dedup layout")
    _check(y, "y", torch.bfloat16, prob.capacity * prob.N, dev)
    _check(topk_weights, "topk_weights", torch.float32, prob.M * prob.topk, dev)
    _check(z, "z", torch.bfloat16, prob.capacity * prob.N, dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_combine_partial(ctypes.byref(s), y.data_ptr(), topk_weights.data_ptr(),
                                         ctypes.byref(l), z.data_ptr(), _stream(y, stream))
    if rc:
        raise MoEError("moe_combine_partial", rc)


def moe_combine_reduce(prob: MoEProblem, z: torch.Tensor, lay: MoELayout, out: torch.Tensor,
                       stream=None) -> None:
    """Token side of the two-level combine: out [M, N] bf16 = sum of the
    token's partition rows of z, in partition order."""
    dev = z.device
    if not prob.dedup:
        raise ValueError("the two-level combine needs a dedup layout")
    _check(z, "z", torch.bfloat16, prob.capacity * prob.N, dev)
    _check(out, "out", torch.bfloat16, prob.M * prob.N, dev)
    _check_layout(prob, lay, dev)
    s, l = prob.struct(), lay.struct()
    rc = _lib.load().moe_combine_reduce(ctypes.byref(s), z.data_ptr(), ctypes.byref(l),
                                        out.data_ptr(), _stream(z, stream))
    if rc:
        raise MoEError("moe_combine_reduce", rc)


@dataclasses.dataclass
class EpPlan:
    """Device arrays of one rank's exchange plan (int32), see ``moe_ep_plan_t``."""
    send_offset: torch.Tensor                          # [W]
    src_offset: torch.Tensor                           # [W]
    recv_count: torch.Tensor                           # [W]
    recv_offset: torch.Tensor                          # [W + 1]
    status: torch.Tensor                               # [1]
    recv_expert_count: Optional[torch.Tensor] = None   # [G]
    recv_block_offset: Optional[torch.Tensor] = None   # [W, G]

    def struct(self) -> _lib.EpPlanStruct:
        def p(t):
            return None if t is None else t.data_ptr()
        return _lib.EpPlanStruct(p(self.send_offset), p(self.src_offset), p(self.recv_count),
                                 p(self.recv_offset), p(self.recv_expert_count),
                                 p(self.recv_block_offset), p(self.status))


def alloc_ep_plan(world: int, G: int = 0, device="cuda") -> EpPlan:
    """Plan arrays for ``world`` ranks; per-expert arrays when ``G`` > 0."""
    i32 = dict(dtype=torch.int32, device=device)
    return EpPlan(torch.empty(world, **i32), torch.empty(world, **i32), torch.empty(world, **i32),
                  torch.empty(world + 1, **i32), torch.empty(1, **i32),
                  torch.empty(G, **i32) if G else None,
                  torch.empty((world, G), **i32) if G else None)


def moe_ep_plan(world: int, rank: int, part_counts: torch.Tensor, plan: EpPlan,
                expert_counts: Optional[torch.Tensor] = None,
                part_of: Optional[torch.Tensor] = None, stream=None) -> None:
    """Rank ``rank``'s offsets for the exchange of dispatch rows among
    ``world`` ranks, from every rank's part_count ``part_counts`` [W, W]
    (and, without dedup, every rank's expert_count ``expert_counts`` [W, G]
    with the placement ``part_of`` [G]), into ``plan``."""
    dev = part_counts.device
    _check(part_counts, "part_counts", torch.int32, world * world, dev)
    for name in ("send_offset", "src_offset", "recv_count"):
        _check(getattr(plan, name), name, torch.int32, world, dev)
    _check(plan.recv_offset, "recv_offset", torch.int32, world + 1, dev)
    _check(plan.status, "status", torch.int32, 1, dev)
    G = 0
    if expert_counts is not None:
        G = expert_counts.numel() // max(world, 1)
        _check(expert_counts, "expert_counts", torch.int32, world * G, dev)
        _check(part_of, "part_of", torch.int32, G, dev)
        _check(plan.recv_expert_count, "recv_expert_count", torch.int32, G, dev)
        _check(plan.recv_block_offset, "recv_block_offset", torch.int32, world * G, dev)
    ps = plan.struct()
    rc = _lib.load().moe_ep_plan(world, rank, G, part_counts.data_ptr(),
                                 None if expert_counts is None else expert_counts.data_ptr(),
                                 None if part_of is None else part_of.data_ptr(),
                                 ctypes.byref(ps), _stream(part_counts, stream))
    if rc:
        raise MoEError("moe_ep_plan", rc)


def ep_all_gather_counts(counts: torch.Tensor, group=None) -> torch.Tensor:
    """The counts exchange: every rank's ``counts`` [K] int32 (its part_count,
    or its expert_count), gathered over the process group into [W, K] in rank
    order, on the device of ``counts`` (NCCL for CUDA tensors, gloo on CPU).
    Every rank of the group must call it, with the same K."""
    import torch.distributed as dist
    W = dist.get_world_size(group)
    parts = [torch.empty_like(counts) for _ in range(W)]
    dist.all_gather(parts, counts.contiguous(), group=group)
    return torch.stack(parts)


@dataclasses.dataclass
class EpPeers:
    """Every rank's buffer as this GPU addresses it, for the expert-parallel
    data plane: a device array of pointers (``table``, int64 [W]), optional
    scale pointers (fp8 dispatch) and the rows each buffer holds.  ``keep``
    holds the tensors the pointers come from, if any, so they stay alive."""
    table: torch.Tensor
    capacity: int
    scale_table: Optional[torch.Tensor] = None
    keep: tuple = ()

    def struct(self) -> _lib.EpPeersStruct:
        return _lib.EpPeersStruct(self.table.data_ptr(),
                                  None if self.scale_table is None else self.scale_table.data_ptr(),
                                  self.capacity)


def ep_peers(rows, capacity: int, scales=None, device="cuda") -> EpPeers:
    """Pointer table from per-rank buffers: tensors on this GPU (local, or
    opened from a peer's memory handle) or raw device addresses (ints), in
    rank order.  Building it copies W pointers to the device once; reuse it
    across steps."""
    def addr(t):
        return int(t) if isinstance(t, int) else t.data_ptr()
    table = torch.tensor([addr(t) for t in rows], dtype=torch.int64).to(device)
    st = None if scales is None else \
        torch.tensor([addr(t) for t in scales], dtype=torch.int64).to(device)
    keep = tuple(t for t in list(rows) + list(scales or []) if isinstance(t, torch.Tensor))
    return EpPeers(table, int(capacity), st, keep)


def moe_ep_dispatch(prob: MoEProblem, x: torch.Tensor, lay: MoELayout, send_offset: torch.Tensor,
                    peers: EpPeers, stream=None) -> None:
    """Push dispatch: every token row of ``x`` stored into each destination
    rank's receive buffer at this rank's ``send_offset`` (from moe_ep_plan)."""
    dev = x.device
    _check(x, "x", torch.bfloat16, prob.M * prob.N, dev)
    _check(send_offset, "send_offset", torch.int32, prob.E_part, dev)
    _check_layout(prob, lay, dev)
    if peers.table.numel() != prob.E_part or (prob.fp8 and peers.scale_table is None):
        raise ValueError("peers: one buffer (and with fp8 one scale buffer) per partition")
    s, l, ps = prob.struct(), lay.struct(), peers.struct()
    rc = _lib.load().moe_ep_dispatch(ctypes.byref(s), x.data_ptr(), ctypes.byref(l),
                                     send_offset.data_ptr(), ctypes.byref(ps), _stream(x, stream))
    if rc:
        raise MoEError("moe_ep_dispatch", rc)


def moe_ep_combine(prob: MoEProblem, y_peers: EpPeers, topk_weights: torch.Tensor, lay: MoELayout,
                   send_offset: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """Pull combine (no dedup): expert outputs gathered from every rank's
    buffer and summed in slot order into ``out`` [M, N] bf16."""
    dev = out.device
    _check(topk_weights, "topk_weights", torch.float32, prob.M * prob.topk, dev)
    _check(out, "out", torch.bfloat16, prob.M * prob.N, dev)
    _check(send_offset, "send_offset", torch.int32, prob.E_part, dev)
    _check_layout(prob, lay, dev)
    if prob.dedup or y_peers.table.numel() != prob.E_part:
        raise ValueError("moe_ep_combine needs a layout without dedup and one buffer per partition")
    s, l, ps = prob.struct(), lay.struct(), y_peers.struct()
    rc = _lib.load().moe_ep_combine(ctypes.byref(s), ctypes.byref(ps), topk_weights.data_ptr(),
                                    ctypes.byref(l), send_offset.data_ptr(), out.data_ptr(),
                                    _stream(out, stream))
    if rc:
        raise MoEError("moe_ep_combine", rc)


def moe_ep_combine_reduce(prob: MoEProblem, z_peers: EpPeers, lay: MoELayout,
                          send_offset: torch.Tensor, out: torch.Tensor, stream=None) -> None:
    """Pull token-side sum of the two-level combine (dedup): each token's
    partition rows gathered from every rank's buffer, summed in partition order."""
    dev = out.device
    _check(out, "out", torch.bfloat16, prob.M * prob.N, dev)
    _check(send_offset, "send_offset", torch.int32, prob.E_part, dev)
    _check_layout(prob, lay, dev)
    if not prob.dedup or z_peers.table.numel() != prob.E_part:
        raise ValueError("moe_ep_combine_reduce needs a dedup layout and one buffer per partition")
    s, l, ps = prob.struct(), lay.struct(), z_peers.struct()
    rc = _lib.load().moe_ep_combine_reduce(ctypes.byref(s), ctypes.byref(ps), ctypes.byref(l),
                                           send_offset.data_ptr(), out.data_ptr(),
                                           _stream(out, stream))
    if rc:
        raise MoEError("moe_ep_combine_reduce", rc)


class MoEBuffers:
    """Caller-side device buffers of one problem at worst-case capacity, and
    the calls of one pass over them (layout -> dispatch -> combine).

    Each call checks the caller's tensors; the buffers of this object are
    checked again only when one of them has been replaced since its last
    check (a few microseconds of host time per call, which matters in
    decode loops)."""

    def __init__(self, prob: MoEProblem, device="cuda"):
        self.prob = prob
        self.device = torch.device(device)
        cap = max(prob.capacity, 1)
        self.layout = alloc_layout(prob, self.device)
        self.workspace = torch.empty(max(layout_workspace_size(prob), 16), dtype=torch.uint8,
                                     device=self.device)
        if prob.fp8:
            self.recv_x = torch.empty((cap, prob.N), dtype=torch.uint8, device=self.device)
            self.recv_scale = torch.empty((cap, prob.N // 128), dtype=torch.float32, device=self.device)
        else:
            self.recv_x = torch.empty((cap, prob.N), dtype=torch.bfloat16, device=self.device)
            self.recv_scale = None
        self.out = torch.empty((max(prob.M, 1), prob.N), dtype=torch.bfloat16, device=self.device)
        self.device = self.out.device          # with its index ("cuda" -> "cuda:0")
        self.z = None
        self.tiles = None
        self._lib = _lib.load()
        self._ps = prob.struct()
        self._ts = None
        self._seen = {}

    def _run(self, name, rc):
        if rc:
            raise MoEError(name, rc)

    def _inputs(self, stream, *checks):
        for t, name, dtype, numel in checks:
            _check(t, name, dtype, numel, self.device)
        return _stream(checks[0][0], stream)

    def _own(self, name, dtype, numel):
        """Device pointer of this object's buffer ``name``, checked again
        whenever the tensor there is not the one checked last."""
        t = getattr(self, name)
        if t is None:
            return None
        key = (id(t), t.data_ptr())
        if self._seen.get(name) != key:
            _check(t, name, dtype, numel, self.device)
            self._seen[name] = key
        return key[1]

    @staticmethod
    def _key(obj):
        """Identity and address of every tensor field of a dataclass (a
        replaced array changes the first, a moved one the second)."""
        return tuple(None if t is None else (id(t), t.data_ptr())
                     for t in (getattr(obj, f.name) for f in dataclasses.fields(obj))
                     if t is None or isinstance(t, torch.Tensor))

    def _lay(self):
        """The layout struct, its arrays checked again when any changed."""
        key = self._key(self.layout)
        if self._seen.get("layout") != key:
            _check_layout(self.prob, self.layout, self.device)
            self._seen["layout"] = key
        return self.layout.struct()

    def _recv(self):
        p = self.prob
        rx = self._own("recv_x", torch.uint8 if p.fp8 else torch.bfloat16, p.capacity * p.N)
        rs = self._own("recv_scale", torch.float32, p.capacity * (p.N // 128)) if p.fp8 else None
        return rx, rs

    def layout_(self, topk_idx, part_of, stream=None):
        p = self.prob
        st = self._inputs(stream, (topk_idx, "topk_idx", torch.int32, p.M * p.topk),
                          (part_of, "part_of", torch.int32, p.G))
        ws = self._own("workspace", torch.uint8, None)
        self._run("moe_layout", self._lib.moe_layout(
            ctypes.byref(self._ps), topk_idx.data_ptr(), part_of.data_ptr(),
            ctypes.byref(self._lay()), ws, self.workspace.numel(), st))

    def dispatch_(self, x, stream=None):
        p = self.prob
        st = self._inputs(stream, (x, "x", torch.bfloat16, p.M * p.N))
        rx, rs = self._recv()
        self._run("moe_dispatch", self._lib.moe_dispatch(
            ctypes.byref(self._ps), x.data_ptr(), ctypes.byref(self._lay()), rx, rs, st))

    def _tiles_for(self, block_m):
        t = self.tiles
        if t is None or t.block_m != block_m:
            self.tiles = t = alloc_expert_tiles(self.prob, block_m, self.device)
            self._ts = t.struct()
        else:
            key = self._key(t)
            if self._seen.get("tiles") != key:     # arrays set by the caller
                _check_tiles(self.prob, t, self.device)
                self._seen["tiles"] = key
            self._ts = t.struct()
        return t

    def layout_dispatch_(self, topk_idx, part_of, x, stream=None, block_m=None):
        """moe_layout_dispatch; ``block_m`` also fills ``self.tiles`` from the
        same kernels."""
        p = self.prob
        st = self._inputs(stream, (x, "x", torch.bfloat16, p.M * p.N),
                          (topk_idx, "topk_idx", torch.int32, p.M * p.topk),
                          (part_of, "part_of", torch.int32, p.G))
        ts = None
        if block_m:
            self._tiles_for(block_m)
            ts = ctypes.byref(self._ts)
        rx, rs = self._recv()
        ws = self._own("workspace", torch.uint8, None)
        self._run("moe_layout_dispatch", self._lib.moe_layout_dispatch(
            ctypes.byref(self._ps), topk_idx.data_ptr(), part_of.data_ptr(), ctypes.byref(self._lay()),
            ws, self.workspace.numel(), x.data_ptr(), rx, rs, ts, st))

    def combine_(self, y, topk_weights, stream=None):
        p = self.prob
        st = self._inputs(stream, (y, "y", torch.bfloat16, p.capacity * p.N),
                          (topk_weights, "topk_weights", torch.float32, p.M * p.topk))
        out = self._own("out", torch.bfloat16, p.M * p.N)
        self._run("moe_combine", self._lib.moe_combine(
            ctypes.byref(self._ps), y.data_ptr(), topk_weights.data_ptr(), ctypes.byref(self._lay()),
            out, st))

    def combine_two_level_(self, y, topk_weights, stream=None):
        """Two-level combine through the dispatch-row buffer ``self.z``
        (allocated on first use)."""
        if self.z is None:
            self.z = torch.empty((max(self.prob.capacity, 1), self.prob.N), dtype=torch.bfloat16,
                                 device=self.device)
        moe_combine_partial(self.prob, y, topk_weights, self.layout, self.z, stream)
        moe_combine_reduce(self.prob, self.z, self.layout, self.out, stream)

    def expert_tiles_(self, part_of, block_m, stream=None):
        """Grouped-GEMM tile metadata of the current layout into ``self.tiles``
        by its own kernel (allocated on first use, or when block_m changes)."""
        moe_expert_tiles(self.prob, part_of, self.layout, self._tiles_for(block_m), stream)

    def step(self, topk_idx, part_of, x, y, topk_weights, stream=None, two_level=False,
             separate=False, block_m=None):
        """layout -> dispatch -> combine; ``separate`` calls moe_layout and
        moe_dispatch instead of moe_layout_dispatch (same results);
        ``block_m`` also builds the grouped-GEMM tile metadata (inside
        moe_layout_dispatch, or by moe_expert_tiles after separate calls)."""
        if separate:
            self.layout_(topk_idx, part_of, stream)
            self.dispatch_(x, stream)
            if block_m:
                self.expert_tiles_(part_of, block_m, stream)
        else:
            self.layout_dispatch_(topk_idx, part_of, x, stream, block_m)
        if two_level:
            self.combine_two_level_(y, topk_weights, stream)
        else:
            self.combine_(y, topk_weights, stream)
        return self.out
