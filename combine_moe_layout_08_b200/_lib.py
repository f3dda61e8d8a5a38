"""ctypes binding of libmoe_layout.so (see include/moe_layout.h).

Argument marshalling only: every step of the path runs in the library's CUDA
kernels.  There is no fallback: if the library is missing and cannot be
built, the first call raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmoe_layout.so")

MOE_OK = 0
MOE_ERR_ARG = 1
MOE_ERR_WORKSPACE = 2
MOE_ERR_CUDA = 3

MOE_ABI_VERSION = 1
MOE_STATUS_BAD_EXPERT = 1
MOE_STATUS_BAD_PART = 2
MOE_STATUS_BAD_ROW = 4
MOE_STATUS_BAD_COUNT = 8

MOE_MAX_G = 1024
MOE_MAX_E_PART = 64
MOE_MAX_TOPK = 32
MOE_MAX_N = 1 << 24
MOE_STATIC_SCRATCH_BYTES = 256 * 1024


class ProblemStruct(ctypes.Structure):
    _fields_ = [("M", ctypes.c_int32), ("N", ctypes.c_int32), ("G", ctypes.c_int32),
                ("topk", ctypes.c_int32), ("E_part", ctypes.c_int32),
                ("dedup", ctypes.c_int32), ("fp8", ctypes.c_int32)]


class LayoutStruct(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "expert_count", "expert_offset", "part_count", "part_offset", "exp_row",
        "disp_token", "disp_row", "exp_to_disp", "status")]


# exported symbol -> (restype, argtypes)
class TilesStruct(ctypes.Structure):
    _fields_ = [("block_m", ctypes.c_int32)] + [
        (n, ctypes.c_void_p) for n in ("tile_first", "tile_expert", "tile_row", "tile_rows")]


class EpPlanStruct(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "send_offset", "src_offset", "recv_count", "recv_offset", "recv_expert_count",
        "recv_block_offset", "status")]


class EpPeersStruct(ctypes.Structure):
    _fields_ = [("rows", ctypes.c_void_p), ("scales", ctypes.c_void_p), ("capacity", ctypes.c_int32)]


SIGNATURES = {
    "moe_abi_version": (ctypes.c_int, []),
    "moe_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "moe_layout_workspace_size": (ctypes.c_size_t, [ctypes.POINTER(ProblemStruct)]),
    "moe_layout": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p, ctypes.c_void_p,
                                  ctypes.POINTER(LayoutStruct), ctypes.c_void_p, ctypes.c_size_t,
                                  ctypes.c_void_p]),
    "moe_layout_static": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                         ctypes.c_void_p, ctypes.POINTER(LayoutStruct),
                                         ctypes.c_void_p]),
    "moe_dispatch": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                    ctypes.POINTER(LayoutStruct), ctypes.c_void_p, ctypes.c_void_p,
                                    ctypes.c_void_p]),
    "moe_layout_dispatch": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.POINTER(LayoutStruct),
                                           ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.c_void_p,
                                           ctypes.POINTER(TilesStruct), ctypes.c_void_p]),
    "moe_layout_dispatch_fused": (ctypes.c_int, [ctypes.POINTER(ProblemStruct)]),
    "moe_expert_tiles_capacity": (ctypes.c_size_t, [ctypes.POINTER(ProblemStruct), ctypes.c_int32]),
    "moe_expert_tiles": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                        ctypes.POINTER(LayoutStruct), ctypes.POINTER(TilesStruct),
                                        ctypes.c_void_p]),
    "moe_combine": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p, ctypes.c_void_p,
                                   ctypes.POINTER(LayoutStruct), ctypes.c_void_p, ctypes.c_void_p]),
    "moe_combine_partial": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                           ctypes.c_void_p, ctypes.POINTER(LayoutStruct),
                                           ctypes.c_void_p, ctypes.c_void_p]),
    "moe_combine_reduce": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                          ctypes.POINTER(LayoutStruct), ctypes.c_void_p,
                                          ctypes.c_void_p]),
    "moe_ep_dispatch": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.c_void_p,
                                       ctypes.POINTER(LayoutStruct), ctypes.c_void_p,
                                       ctypes.POINTER(EpPeersStruct), ctypes.c_void_p]),
    "moe_ep_combine": (ctypes.c_int, [ctypes.POINTER(ProblemStruct), ctypes.POINTER(EpPeersStruct),
                                      ctypes.c_void_p, ctypes.POINTER(LayoutStruct), ctypes.c_void_p,
                                      ctypes.c_void_p, ctypes.c_void_p]),
    "moe_ep_combine_reduce": (ctypes.c_int, [ctypes.POINTER(ProblemStruct),
                                             ctypes.POINTER(EpPeersStruct),
                                             ctypes.POINTER(LayoutStruct), ctypes.c_void_p,
                                             ctypes.c_void_p, ctypes.c_void_p]),
    "moe_ep_plan": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int32, ctypes.c_int32, ctypes.c_void_p,
                                   ctypes.c_void_p, ctypes.c_void_p, ctypes.POINTER(EpPlanStruct),
                                   ctypes.c_void_p]),
}

_lock = threading.Lock()
_lib = None


def load():
    """Load the in-tree library (building it once if it is absent)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(LIB_PATH):
            from . import build as _build
            _build.build()
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m combine_moe_layout_08_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        if L.moe_abi_version() != MOE_ABI_VERSION:
            raise RuntimeError(f"{LIB_PATH}: ABI version {L.moe_abi_version()}, the binding "
                               f"expects {MOE_ABI_VERSION}; rebuild the library")
        _lib = L
        return L


class MoEError(RuntimeError):
    def __init__(self, fn: str, code: int):
        msg = load().moe_status_string(code).decode()
        super().__init__(f"{fn} returned {code}: {msg}")
        self.code = code
