"""Helpers of the GPU parity tests: run the CUDA path through the C ABI on
seeded inputs and compare it with the oracle element by element."""
from __future__ import annotations

import numpy as np
import torch

import combine_moe_layout_08_b200 as moe
import oracle
import workloads as W

POISON_I32 = -7
POISON_BYTE = 0xA5


def problem_of(w: W.Workload) -> moe.MoEProblem:
    return moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)


def to_dev(a, dev="cuda"):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dev)


def poisoned_buffers(prob: moe.MoEProblem, dev="cuda") -> moe.MoEBuffers:
    b = moe.MoEBuffers(prob, dev)
    for t in (b.layout.expert_count, b.layout.expert_offset, b.layout.part_count,
              b.layout.part_offset, b.layout.exp_row, b.layout.disp_token, b.layout.status,
              b.layout.disp_row, b.layout.exp_to_disp):
        if t is not None:
            t.fill_(POISON_I32)
    b.recv_x.view(torch.uint8).fill_(POISON_BYTE)
    if b.recv_scale is not None:
        b.recv_scale.view(torch.uint8).fill_(POISON_BYTE)
    b.out.view(torch.uint8).fill_(POISON_BYTE)
    b.workspace.fill_(0x5A)
    return b


def run_path(prob, idx, part_of, weights, x, y, dev="cuda") -> moe.MoEBuffers:
    """layout -> dispatch -> combine on the device; returns the buffers."""
    b = poisoned_buffers(prob, dev)
    b.layout_(to_dev(idx, dev), to_dev(part_of, dev))
    b.dispatch_(x)
    b.combine_(y, to_dev(weights, dev))
    torch.cuda.synchronize()
    return b


def np_i32(t) -> np.ndarray:
    return t.detach().cpu().numpy()


def compare_layout(b: moe.MoEBuffers, ref: dict, prob: moe.MoEProblem):
    L = b.layout
    R_exp, R_disp = ref["R_exp"], ref["R_disp"]
    assert int(np_i32(L.status)[0]) == ref["status"]
    np.testing.assert_array_equal(np_i32(L.expert_count), ref["expert_count"])
    np.testing.assert_array_equal(np_i32(L.expert_offset), ref["expert_offset"])
    np.testing.assert_array_equal(np_i32(L.part_count), ref["part_count"])
    np.testing.assert_array_equal(np_i32(L.part_offset), ref["part_offset"])
    M, topk = prob.M, prob.topk
    np.testing.assert_array_equal(np_i32(L.exp_row)[:M * topk].reshape(M, topk), ref["exp_row"])
    dt = np_i32(L.disp_token)
    np.testing.assert_array_equal(dt[:R_disp], ref["disp_token"])
    assert np.all(dt[R_disp:prob.capacity] == POISON_I32), "rows past R_disp must stay untouched"
    if prob.dedup:
        np.testing.assert_array_equal(np_i32(L.disp_row)[:M * prob.E_part].reshape(M, prob.E_part),
                                      ref["disp_row"])
        e2d = np_i32(L.exp_to_disp)
        np.testing.assert_array_equal(e2d[:R_exp], ref["exp_to_disp"])
        assert np.all(e2d[R_exp:prob.capacity] == POISON_I32)


def ulp_distance_bf16(a_bits: np.ndarray, b_bits: np.ndarray) -> np.ndarray:
    """Distance in bf16 steps; +0 and -0 both map to 0."""
    def key(b):
        v = np.asarray(b, np.int32)
        mag = v & 0x7FFF
        return np.where(v & 0x8000, -mag, mag)
    return np.abs(key(a_bits) - key(b_bits))


def compare_dispatch_rows(b: moe.MoEBuffers, prob, x_bits, disp_token, rows=None):
    """Dispatch rows (all of [0, R_disp), or the sample ``rows``) bit-exact."""
    R_disp = disp_token.shape[0]
    sel = np.arange(R_disp) if rows is None else np.asarray(rows, np.int64)
    if sel.size == 0:
        return
    idx_t = torch.from_numpy(sel).to(b.recv_x.device)
    got = b.recv_x[idx_t].cpu()
    # only the token rows the sample needs travel to the oracle
    toks = disp_token[sel]
    uniq, inv = np.unique(toks, return_inverse=True)
    x_sub = x_bits[uniq]
    if prob.fp8:
        q, s = oracle.dispatch(x_sub, inv.astype(np.int32), True)
        np.testing.assert_array_equal(got.numpy(), q)
        gs = b.recv_scale[idx_t].cpu().numpy()
        np.testing.assert_array_equal(gs.view(np.uint32), s.view(np.uint32))
    else:
        want = oracle.dispatch(x_sub, inv.astype(np.int32), False)
        np.testing.assert_array_equal(got.view(torch.int16).numpy().view(np.uint16), want)


def untouched_rows_ok(b: moe.MoEBuffers, R_disp: int):
    if R_disp >= b.prob.capacity:
        return
    tail = b.recv_x[R_disp:].view(torch.uint8)
    assert bool((tail == POISON_BYTE).all()), "dispatch wrote past R_disp"
    if b.recv_scale is not None:
        assert bool((b.recv_scale[R_disp:].view(torch.uint8) == POISON_BYTE).all())


def compare_combine(b: moe.MoEBuffers, prob, y_dev, weights, exp_row, tokens=None, max_ulp=1):
    """out rows (all, or the sample ``tokens``) within max_ulp bf16 steps of
    the oracle; returns the number of elements that differ at all."""
    M, topk = exp_row.shape
    tok = np.arange(M) if tokens is None else np.asarray(tokens, np.int64)
    if tok.size == 0:
        return 0
    er = exp_row[tok]                                     # [n, topk]
    valid = er >= 0
    rows = np.where(valid, er, 0).ravel()
    y_sub = oracle.bf16_bits(y_dev[torch.from_numpy(rows).to(y_dev.device)])
    er_sub = np.where(valid, np.arange(rows.size).reshape(er.shape), -1).astype(np.int32)
    want = oracle.combine(y_sub, weights[tok], er_sub)
    got = oracle.bf16_bits(b.out[torch.from_numpy(tok).to(b.out.device)])
    d = ulp_distance_bf16(got, want)
    assert d.max(initial=0) <= max_ulp, f"combine differs by {d.max()} bf16 steps"
    return int(np.count_nonzero(got != want))


def compare_two_level(b: moe.MoEBuffers, prob, y_dev, gates, idx, part_of, ref, tokens=None,
                      max_ulp=1):
    """Two-level combine: the partition rows z (all, or those of the sample
    ``tokens``) bit-exact, and out within max_ulp bf16 steps of the oracle
    (which runs on a compact copy of the sampled tokens); returns the number
    of out elements that differ at all."""
    M, topk = idx.shape
    E = prob.E_part
    tok = np.arange(M) if tokens is None else np.asarray(tokens, np.int64)
    n = tok.size
    er = ref["exp_row"][tok]
    dr = ref["disp_row"][tok]
    valid = er >= 0
    rows = np.where(valid, er, 0).ravel()
    y_sub = oracle.bf16_bits(y_dev[torch.from_numpy(rows).to(y_dev.device)])
    er_sub = np.where(valid, np.arange(n * topk).reshape(n, topk), -1).astype(np.int32)
    dvalid = dr >= 0
    dr_sub = np.where(dvalid, np.arange(n * E).reshape(n, E), -1).astype(np.int32)
    lay_sub = dict(exp_row=er_sub, disp_row=dr_sub, R_disp=n * E)
    z_ref = oracle.combine_partial(y_sub, gates[tok], idx[tok], part_of, lay_sub)
    out_ref = oracle.combine_reduce(z_ref, dr_sub)
    z_got = oracle.bf16_bits(b.z[torch.from_numpy(dr[dvalid].astype(np.int64)).to(b.z.device)])
    np.testing.assert_array_equal(z_got, z_ref[dr_sub[dvalid]])
    got = oracle.bf16_bits(b.out[torch.from_numpy(tok).to(b.out.device)])
    d = ulp_distance_bf16(got, out_ref)
    assert d.max(initial=0) <= max_ulp, f"two-level combine differs by {d.max()} bf16 steps"
    return int(np.count_nonzero(got != out_ref))


# ---------------------------------------------------------------------------
# element-by-element comparison of a large batch, in chunks
# ---------------------------------------------------------------------------
def run_chunks(jobs, workers=None, in_flight=None):
    """``jobs`` yields (label, check, args): the device -> host gathers run
    in the caller's thread as the generator advances, each ``check(*args)``
    (oracle + comparison, plain C through ctypes, which releases the GIL) in
    a pool of threads.  At most ``in_flight`` gathered chunks are held at
    once.  Returns the results in order; the first failing check raises."""
    import os
    import threading
    from concurrent.futures import ThreadPoolExecutor
    workers = workers or max(1, min(32, len(os.sched_getaffinity(0))))
    gate = threading.BoundedSemaphore(in_flight or workers + 2)
    futs = []

    def wrapped(label, check, args):
        try:
            return check(*args)
        except AssertionError as e:
            raise AssertionError(f"{label}: {e}") from None
        finally:
            gate.release()

    with ThreadPoolExecutor(workers) as ex:
        for label, check, args in jobs:
            gate.acquire()
            futs.append(ex.submit(wrapped, label, check, args))
        return [f.result() for f in futs]


def _check_dispatch_chunk(x_bits, dt, fp8, got, got_scale):
    if fp8:
        q, s = oracle.dispatch(x_bits, dt, True)
        np.testing.assert_array_equal(got, q)
        np.testing.assert_array_equal(got_scale.view(np.uint32), s.view(np.uint32))
    else:
        np.testing.assert_array_equal(got, oracle.dispatch(x_bits, dt, False))
    return dt.shape[0]


def dispatch_all_rows(b: moe.MoEBuffers, prob, x_bits, disp_token, rows_per_chunk=8192):
    """Every dispatch row [0, R_disp) (bytes, and scales with FP8) bit-exact
    against the oracle; returns the number of rows compared."""
    R = disp_token.shape[0]

    def jobs():
        for r0 in range(0, R, rows_per_chunk):
            r1 = min(R, r0 + rows_per_chunk)
            got = b.recv_x[r0:r1]
            got = got.cpu().numpy() if prob.fp8 else \
                got.view(torch.int16).cpu().numpy().view(np.uint16)
            gs = b.recv_scale[r0:r1].cpu().numpy() if prob.fp8 else None
            yield f"dispatch rows [{r0}, {r1})", _check_dispatch_chunk, \
                (x_bits, disp_token[r0:r1], prob.fp8, got, gs)

    return sum(run_chunks(jobs()))


def _check_combine_chunk(y_sub, gates, er_sub, got, max_ulp):
    want = oracle.combine(y_sub, gates, er_sub)
    d = ulp_distance_bf16(got, want)
    assert d.max(initial=0) <= max_ulp, f"combine differs by {d.max()} bf16 steps"
    return int(np.count_nonzero(got != want))


def _gather_rows(t: torch.Tensor, rows: np.ndarray) -> np.ndarray:
    return oracle.bf16_bits(t[torch.from_numpy(rows.astype(np.int64)).to(t.device)])


def combine_all_tokens(b: moe.MoEBuffers, y_dev, gates, exp_row, tokens_per_chunk=1024, max_ulp=1):
    """Every out row within max_ulp bf16 steps of the oracle; returns the
    number of elements that differ at all (expected 0)."""
    M, topk = exp_row.shape

    def jobs():
        for t0 in range(0, M, tokens_per_chunk):
            t1 = min(M, t0 + tokens_per_chunk)
            er = exp_row[t0:t1]
            valid = er >= 0
            y_sub = _gather_rows(y_dev, np.where(valid, er, 0).ravel())
            er_sub = np.where(valid, np.arange(er.size).reshape(er.shape), -1).astype(np.int32)
            got = oracle.bf16_bits(b.out[t0:t1])
            yield f"combine tokens [{t0}, {t1})", _check_combine_chunk, \
                (y_sub, gates[t0:t1], er_sub, got, max_ulp)

    return sum(run_chunks(jobs()))


def _check_two_level_chunk(y_sub, gates, idx, part_of, er_sub, dr_sub, z_got, z_sel, got, max_ulp):
    n, E = dr_sub.shape
    lay_sub = dict(exp_row=er_sub, disp_row=dr_sub, R_disp=n * E)
    z_ref = oracle.combine_partial(y_sub, gates, idx, part_of, lay_sub)
    out_ref = oracle.combine_reduce(z_ref, dr_sub)
    np.testing.assert_array_equal(z_got, z_ref[z_sel])
    d = ulp_distance_bf16(got, out_ref)
    assert d.max(initial=0) <= max_ulp, f"two-level combine differs by {d.max()} bf16 steps"
    return int(np.count_nonzero(got != out_ref))


def two_level_all_tokens(b: moe.MoEBuffers, prob, y_dev, gates, idx, part_of, ref,
                         tokens_per_chunk=1024, max_ulp=1):
    """Two-level combine of every token: all z rows bit-exact, every out row
    within max_ulp bf16 steps; returns the out elements that differ."""
    M, topk = idx.shape
    E = prob.E_part

    def jobs():
        for t0 in range(0, M, tokens_per_chunk):
            t1 = min(M, t0 + tokens_per_chunk)
            n = t1 - t0
            er = ref["exp_row"][t0:t1]
            dr = ref["disp_row"][t0:t1]
            valid = er >= 0
            y_sub = _gather_rows(y_dev, np.where(valid, er, 0).ravel())
            er_sub = np.where(valid, np.arange(n * topk).reshape(n, topk), -1).astype(np.int32)
            dvalid = dr >= 0
            dr_sub = np.where(dvalid, np.arange(n * E).reshape(n, E), -1).astype(np.int32)
            z_got = _gather_rows(b.z, dr[dvalid])
            got = oracle.bf16_bits(b.out[t0:t1])
            yield f"two-level tokens [{t0}, {t1})", _check_two_level_chunk, \
                (y_sub, gates[t0:t1], idx[t0:t1], part_of, er_sub, dr_sub, z_got, dr_sub[dvalid],
                 got, max_ulp)

    return sum(run_chunks(jobs()))
