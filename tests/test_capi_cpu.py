"""The C ABI without a GPU: the library builds and loads, exports every
function include/moe_layout.h declares, and rejects invalid calls on the host
before any CUDA call (fake device pointers never reach a kernel: these tests
skip on a machine with a GPU, where the GPU tests cover the same checks with
real buffers)."""
import ctypes
import os
import re
import subprocess

import pytest
import torch

from combine_moe_layout_08_b200 import _lib, build as libbuild

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "moe_layout.h")


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(moe_\w+)\s*\(", src, flags=re.M)))


@pytest.fixture(scope="module")
def L():
    libbuild.build()
    return _lib.load()


def test_header_declares_the_path():
    names = declared_functions()
    for n in ("moe_layout", "moe_dispatch", "moe_combine", "moe_layout_workspace_size",
              "moe_status_string", "moe_abi_version"):
        assert n in names


def test_exports_every_declared_symbol(L):
    for n in declared_functions():
        assert hasattr(L, n), n
    assert set(declared_functions()) <= set(_lib.SIGNATURES)


def test_dynamic_symbol_table():
    out = subprocess.run(["nm", "-D", "--defined-only", _lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert set(declared_functions()) <= exported


def test_version_and_strings(L):
    assert L.moe_abi_version() == 1
    for c in range(5):
        assert L.moe_status_string(c)


def P(**kw):
    d = dict(M=128, N=7168, G=256, topk=8, E_part=8, dedup=0, fp8=0)
    d.update(kw)
    return _lib.ProblemStruct(**d)


def test_workspace_size(L):
    from combine_moe_layout_08_b200 import _lib as l2  # noqa: F401
    ws = L.moe_layout_workspace_size(ctypes.byref(P()))
    assert ws > 0 and ws % 256 == 0
    big = L.moe_layout_workspace_size(ctypes.byref(P(M=65536, dedup=1)))
    assert big > ws
    # one row per tile (about one tile per SM): G expert counts, E partition
    # counts (dedup), two invalid-input counters, padded to 4 ints
    T = max(128, ((65536 + 147) // 148 + 31) // 32 * 32)
    nt = (65536 + T - 1) // T
    W = (256 + 8 + 2 + 3) // 4 * 4
    assert big == ((nt * W * 4 + 255) // 256) * 256
    for bad in (P(N=7), P(G=0), P(G=1025), P(topk=0), P(topk=33), P(E_part=0), P(E_part=65),
                P(M=-1), P(fp8=1, N=7176), P(dedup=2), P(M=1 << 28, topk=8),
                P(N=(1 << 24) + 8)):
        assert L.moe_layout_workspace_size(ctypes.byref(bad)) == 0
    assert L.moe_layout_workspace_size(None) == 0
    assert L.moe_layout_workspace_size(ctypes.byref(P(N=1 << 24))) > 0   # the largest N


def _expected_workspace(M, G, E, dedup):
    """One row per tile of T tokens, T = max(128, ceil(M / 148) rounded up to
    32), rows of G (+ E with dedup) + 2 ints padded to 4, rounded to 256 B;
    Python integers, so nothing overflows."""
    T = max(128, -(-(-(-M // 148)) // 32) * 32)
    nt = max(1, -(-M // T))
    W = -(-(G + (E if dedup else 0) + 2) // 4) * 4
    return -(-(nt * W * 4) // 256) * 256, nt


@pytest.mark.parametrize("topk,E,dedup", [(1, 1, 0), (1, 1, 1), (2, 1, 0), (1, 2, 1)])
def test_workspace_size_at_the_largest_batch(L, topk, E, dedup):
    """M up to the admitted limit (M*topk and M*E_part below 2^31): the tile
    arithmetic must not overflow 32 bits, and one past the limit is refused."""
    top = (1 << 31) - 1
    M = min(top // topk, top // E)
    for G in (1, 256, 1024):
        want, nt = _expected_workspace(M, G, E, dedup)
        assert nt == 148
        got = L.moe_layout_workspace_size(ctypes.byref(P(M=M, N=8, G=G, topk=topk, E_part=E,
                                                         dedup=dedup)))
        assert got == want, (M, G, got, want)
    assert L.moe_layout_workspace_size(ctypes.byref(P(M=M + 1, N=8, G=8, topk=topk, E_part=E,
                                                      dedup=dedup))) == 0
    # every M just below the limit, including those where M + 147 passes 2^31
    for m in (M - 1, M - 100, M - 147, M - 148, M - 200, min(M, (1 << 31) - 148 * 32)):
        want, _ = _expected_workspace(m, 64, E, dedup)
        got = L.moe_layout_workspace_size(ctypes.byref(P(M=m, N=8, G=64, topk=topk, E_part=E,
                                                         dedup=dedup)))
        assert got == want, (m, got, want)


no_gpu = pytest.mark.skipif(torch.cuda.is_available(), reason="fake pointers only without a GPU")

FAKE = 0x7f0000000000  # never dereferenced: every call below fails validation


def fake_layout(**over):
    f = {n: FAKE + 4096 * i for i, (n, _) in enumerate(_lib.LayoutStruct._fields_)}
    f.update(over)
    return _lib.LayoutStruct(**f)


@no_gpu
def test_layout_rejects_bad_arguments(L):
    ok_ws = L.moe_layout_workspace_size(ctypes.byref(P()))
    lay = fake_layout()
    # invalid problems
    for bad in (P(N=12), P(G=2000), P(topk=40), P(E_part=100), P(fp8=1, N=136)):
        assert L.moe_layout(ctypes.byref(bad), FAKE, FAKE, ctypes.byref(lay), FAKE, 1 << 30, None) == 1
    assert L.moe_layout(None, FAKE, FAKE, ctypes.byref(lay), FAKE, ok_ws, None) == 1
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, None, FAKE, ok_ws, None) == 1
    # missing / misaligned arrays
    assert L.moe_layout(ctypes.byref(P()), FAKE, None, ctypes.byref(lay), FAKE, ok_ws, None) == 1
    assert L.moe_layout(ctypes.byref(P()), FAKE + 2, FAKE, ctypes.byref(lay), FAKE, ok_ws, None) == 1
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, ctypes.byref(fake_layout(status=None)),
                        FAKE, ok_ws, None) == 1
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, ctypes.byref(fake_layout(exp_row=FAKE + 1)),
                        FAKE, ok_ws, None) == 1
    # dedup needs disp_row and exp_to_disp
    assert L.moe_layout(ctypes.byref(P(dedup=1)), FAKE, FAKE, ctypes.byref(fake_layout(disp_row=None)),
                        FAKE, 1 << 30, None) == 1
    # workspace
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, ctypes.byref(lay), FAKE, ok_ws - 1, None) == 2
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, ctypes.byref(lay), None, ok_ws, None) == 2
    assert L.moe_layout(ctypes.byref(P()), FAKE, FAKE, ctypes.byref(lay), FAKE + 8, ok_ws, None) == 2


@no_gpu
def test_dispatch_combine_reject_bad_arguments(L):
    lay = fake_layout()
    p = ctypes.byref(P())
    assert L.moe_dispatch(p, None, ctypes.byref(lay), FAKE, None, None) == 1
    assert L.moe_dispatch(p, FAKE + 8, ctypes.byref(lay), FAKE, None, None) == 1
    assert L.moe_dispatch(p, FAKE, ctypes.byref(lay), FAKE + 4, None, None) == 1
    assert L.moe_dispatch(ctypes.byref(P(fp8=1)), FAKE, ctypes.byref(lay), FAKE, None, None) == 1
    assert L.moe_dispatch(p, FAKE, None, FAKE, None, None) == 1
    assert L.moe_combine(p, None, FAKE, ctypes.byref(lay), FAKE, None) == 1
    assert L.moe_combine(p, FAKE, None, ctypes.byref(lay), FAKE, None) == 1
    assert L.moe_combine(p, FAKE, FAKE + 2, ctypes.byref(lay), FAKE, None) == 1
    assert L.moe_combine(p, FAKE, FAKE, ctypes.byref(lay), FAKE + 8, None) == 1
    assert L.moe_combine(ctypes.byref(P(N=0)), FAKE, FAKE, ctypes.byref(lay), FAKE, None) == 1
    # the two-level combine needs a dedup problem
    assert L.moe_combine_partial(p, FAKE, FAKE, ctypes.byref(lay), FAKE, None) == 1
    assert L.moe_combine_reduce(p, FAKE, ctypes.byref(lay), FAKE, None) == 1
    pd = ctypes.byref(P(dedup=1))
    assert L.moe_combine_partial(pd, FAKE + 4, FAKE, ctypes.byref(lay), FAKE, None) == 1
    assert L.moe_combine_reduce(pd, FAKE, ctypes.byref(lay), FAKE + 8, None) == 1


def test_fused_schedule_query(L):
    """moe_layout_dispatch takes one kernel for small batches only."""
    f = lambda **kw: L.moe_layout_dispatch_fused(ctypes.byref(P(**kw)))
    assert f(M=128) == 1 and f(M=1) == 1 and f(M=512) == 1
    assert f(M=513) == 0 and f(M=4096) == 0 and f(M=0) == 0
    assert f(M=2048, topk=2) == 1 and f(M=2049, topk=2) == 0
    assert f(N=12) == 0 and L.moe_layout_dispatch_fused(None) == 0


@no_gpu
def test_layout_dispatch_rejects_bad_arguments(L):
    lay = fake_layout()
    ws = L.moe_layout_workspace_size(ctypes.byref(P()))
    call = lambda prob, idx=FAKE, po=FAKE, lay_=lay, w=FAKE, wb=ws, x=FAKE, r=FAKE, sc=None, t=None: \
        L.moe_layout_dispatch(ctypes.byref(prob), idx, po, ctypes.byref(lay_) if lay_ else None,
                              w, wb, x, r, sc, ctypes.byref(t) if t else None, None)
    assert call(P(N=12)) == 1
    assert call(P(), idx=FAKE + 2) == 1
    assert call(P(), po=None) == 1
    assert call(P(), x=FAKE + 8) == 1
    assert call(P(), r=None) == 1
    assert call(P(fp8=1)) == 1                       # fp8 needs recv_scale
    assert call(P(dedup=1), lay_=fake_layout(exp_to_disp=None)) == 1
    assert call(P(), wb=ws - 1) == 2
    assert call(P(), w=FAKE + 8) == 2
    # an invalid tile request
    assert call(P(), t=_lib.TilesStruct(0, FAKE, FAKE, FAKE, FAKE)) == 1
    assert call(P(), t=_lib.TilesStruct(128, FAKE, None, FAKE, FAKE)) == 1
    assert call(P(), t=_lib.TilesStruct(128, FAKE, FAKE, FAKE + 2, FAKE)) == 1


def test_expert_tiles_capacity(L):
    cap = lambda bm, **kw: L.moe_expert_tiles_capacity(ctypes.byref(P(**kw)), bm)
    assert cap(128) == (128 * 8 + 127) // 128 + 256
    assert cap(1) == 128 * 8 + 256
    assert cap(0) == 0 and cap(-3) == 0 and cap(128, N=12) == 0
    assert cap(7, M=0) == 256


@no_gpu
def test_expert_tiles_rejects_bad_arguments(L):
    lay = fake_layout()
    p = ctypes.byref(P())
    T = lambda bm, *arrs: ctypes.byref(_lib.TilesStruct(bm, *arrs))
    ok = (FAKE, FAKE + 64, FAKE + 128, FAKE + 192)
    assert L.moe_expert_tiles(p, FAKE, ctypes.byref(lay), T(0, *ok), None) == 1
    assert L.moe_expert_tiles(p, None, ctypes.byref(lay), T(64, *ok), None) == 1
    assert L.moe_expert_tiles(p, FAKE, None, T(64, *ok), None) == 1
    assert L.moe_expert_tiles(p, FAKE, ctypes.byref(lay), T(64, FAKE, FAKE + 2, FAKE, FAKE), None) == 1
    assert L.moe_expert_tiles(p, FAKE, ctypes.byref(lay), T(64, FAKE, FAKE, FAKE, None), None) == 1
    assert L.moe_expert_tiles(p, FAKE, ctypes.byref(lay), None, None) == 1


def test_python_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    """No silent fallback: a missing library that cannot be built raises."""
    monkeypatch.setattr(_lib, "_lib", None)
    monkeypatch.setattr(_lib, "LIB_PATH", str(tmp_path / "absent.so"))
    import combine_moe_layout_08_b200.build as b
    monkeypatch.setattr(b, "build", lambda *a, **k: str(tmp_path / "absent.so"))
    with pytest.raises(RuntimeError):
        _lib.load()


@no_gpu
def test_ep_plan_rejects_bad_arguments(L):
    def plan(**over):
        f = {n: FAKE + 4096 * (i + 1) for i, (n, _) in enumerate(_lib.EpPlanStruct._fields_)}
        f.update(over)
        return ctypes.byref(_lib.EpPlanStruct(**f))
    ok = plan()
    for world, rank in ((0, 0), (65, 0), (4, 4), (4, -1)):
        assert L.moe_ep_plan(world, rank, 8, FAKE, None, None, ok, None) == 1
    assert L.moe_ep_plan(4, 0, 8, None, None, None, ok, None) == 1             # no counts
    assert L.moe_ep_plan(4, 0, 8, FAKE + 2, None, None, ok, None) == 1         # misaligned
    assert L.moe_ep_plan(4, 0, 8, FAKE, None, None, None, None) == 1           # no plan
    assert L.moe_ep_plan(4, 0, 8, FAKE, None, None, plan(status=None), None) == 1
    assert L.moe_ep_plan(4, 0, 8, FAKE, None, None, plan(recv_offset=FAKE + 1), None) == 1
    # with expert counts: G in range, placement and per-expert arrays required
    assert L.moe_ep_plan(4, 0, 0, FAKE, FAKE, FAKE, ok, None) == 1
    assert L.moe_ep_plan(4, 0, 1025, FAKE, FAKE, FAKE, ok, None) == 1
    assert L.moe_ep_plan(4, 0, 8, FAKE, FAKE, None, ok, None) == 1
    assert L.moe_ep_plan(4, 0, 8, FAKE, FAKE, FAKE, plan(recv_block_offset=None), None) == 1


C_HOST = r"""
#include <stdio.h>
#include "moe_layout.h"

int main(void) {
    moe_problem_t p = {4096, 7168, 256, 8, 8, 0, 0};
    moe_problem_t bad = {4096, 7, 256, 8, 8, 0, 0};
    moe_layout_t lay = {0};
    moe_tiles_t tiles = {0};
    if (moe_abi_version() != MOE_ABI_VERSION) return 1;
    if (moe_layout_workspace_size(&p) == 0 || moe_layout_workspace_size(&bad) != 0) return 2;
    if (moe_expert_tiles_capacity(&p, 128) != (4096 * 8 + 127) / 128 + 256) return 3;
    if (moe_layout_dispatch_fused(&p) != 0) return 4;
    if (moe_status_string(MOE_ERR_ARG)[0] == 0) return 5;
    /* invalid calls fail on the host, before any CUDA call */
    if (moe_layout(&bad, 0, 0, &lay, 0, 0, 0) != MOE_ERR_ARG) return 6;
    if (moe_expert_tiles(&p, 0, &lay, &tiles, 0) != MOE_ERR_ARG) return 7;
    (void)moe_layout_static; (void)moe_dispatch; (void)moe_combine;
    (void)moe_combine_partial; (void)moe_combine_reduce; (void)moe_ep_plan;
    {
        moe_ep_plan_t plan = {0};
        /* an invalid call fails on the host: rank outside [0, world) */
        if (moe_ep_plan(2, 2, 8, 0, 0, 0, &plan, 0) != MOE_ERR_ARG) return 8;
    }
    printf("ok\n");
    return 0;
}
"""


def test_plain_c_host_compiles_links_and_calls(tmp_path):
    """The header is plain C99, and a C program links the library and calls
    the entry points that need no GPU."""
    libbuild.build()
    src = tmp_path / "host.c"
    exe = tmp_path / "host"
    src.write_text(C_HOST)
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["gcc", "-std=c99", "-Wall", "-Werror", "-I", os.path.dirname(HEADER), str(src),
                    "-L", lib_dir, "-lmoe_layout", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)


def test_header_compiles_as_cpp(tmp_path):
    """The same host program as C++17: the header's extern "C" block keeps
    the names unmangled, so it links against the library."""
    libbuild.build()
    src = tmp_path / "host.cpp"
    exe = tmp_path / "host_cpp"
    src.write_text(C_HOST)
    lib_dir = os.path.dirname(_lib.LIB_PATH)
    subprocess.run(["g++", "-std=c++17", "-Wall", "-Werror", "-I", os.path.dirname(HEADER),
                    str(src), "-L", lib_dir, "-lmoe_layout", f"-Wl,-rpath,{lib_dir}", "-o", str(exe)],
                   check=True, capture_output=True)
    out = subprocess.run([str(exe)], capture_output=True, text=True)
    assert out.returncode == 0 and out.stdout.strip() == "ok", (out.returncode, out.stderr)


def test_python_constants_match_the_header():
    src = open(HEADER).read()
    defs = {k: v.strip() for k, v in re.findall(r"#define (MOE_\w+)[ \t]+([^/\n]+)", src)}
    for name in ("MOE_MAX_G", "MOE_MAX_E_PART", "MOE_MAX_TOPK", "MOE_MAX_N", "MOE_STATUS_BAD_EXPERT",
                 "MOE_STATUS_BAD_PART", "MOE_STATUS_BAD_ROW", "MOE_STATUS_BAD_COUNT",
                 "MOE_ABI_VERSION"):
        assert eval(defs[name]) == getattr(_lib, name), (name, defs[name])   # integer literals


def test_static_scratch_fit_rule(L):
    """moe_layout_static fits every M when G + (dedup ? E_part : 0) <= 438 (the
    rule its header states) and not beyond."""
    cap = 256 * 1024

    def size(G, E, dedup):
        M = ((1 << 31) - 1) // E                   # the largest batch admitted (M * E_part < 2^31)
        n = L.moe_layout_workspace_size(ctypes.byref(P(M=M, N=8, G=G, topk=1, E_part=E, dedup=dedup)))
        assert n > 0
        return n
    for G, E, dedup in ((438, 1, 0), (430, 8, 1), (374, 64, 1), (256, 8, 1), (438, 64, 0)):
        assert size(G, E, dedup) <= cap, (G, E, dedup)
    for G, E, dedup in ((439, 1, 0), (431, 8, 1), (375, 64, 1)):
        assert size(G, E, dedup) > cap, (G, E, dedup)
