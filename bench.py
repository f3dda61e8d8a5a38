#!/usr/bin/env python
"""Benchmark of the MoE dispatch / combine path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--schedule auto|separate] [--tiles BM]
                    [--combine one-level|two-level] [--latency-sweep]

One step = one pass of the whole path over one batch: routing layout ->
dispatch permute -> combine (libmoe_layout.so, through its C ABI), on the
largest workload by default: the prefill batch of M = 65536 tokens, N =
7168, G = 256, topk = 8, E_part = 8, routing 50% uniform / 50% Zipf(1.2),
per-partition dedup and the FP8 dispatch.  Inputs are resident in HBM when
the timed region starts.  Each
step is one CUDA-graph replay with events at its two ends on the device;
a second graph of the same step with events between its parts gives the
per-kernel breakdown.  L2 is flushed between steps (256 MiB written, then
256 MiB read, untimed).

Printed (rank 0, one JSON line): value = algorithmic HBM bytes of the whole
path per second (GB/s) over all ranks; tokens/s; per-kernel times; the
roofline of the dominant kernel against the measured copy bandwidth; the
end-to-end figure through the public API with host buffers (host->device
copies of the inputs and device->host copy of the output in the timed
region); the CPU oracle timed on the host (rank 0, N = 1).

Multi-GPU: one process per GPU under torchrun; every rank runs its own
batch (data-parallel replicas, no collective on the data path); the time is
the max over ranks.  ``--impl reference`` times the CPU oracle instead.
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import re
import statistics
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import workloads as W  # noqa: E402

DEFAULT_WORKLOAD = "prefill-M65536-mix-dedup-fp8"
# batch sizes of the decode latency sweep: the M column of the latency table
# of Triton-distributed issue #117 ("Results (Latency in us)")
SWEEP_M = (2, 4, 8, 16, 32, 64, 128, 256, 512)
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


# ---------------------------------------------------------------------------
# algorithmic bytes (HBM traffic the path cannot avoid), per kernel
# ---------------------------------------------------------------------------
def algorithmic_bytes(w: W.Workload, R_exp: int, R_disp: int, two_level: bool = False) -> dict:
    M, N, G, k, E = w.M, w.N, w.G, w.topk, w.E_part
    layout = 4 * M * k + 4 * G + 4 * M * k + 4 * R_disp + 4 * (2 * G + 2 * E + 2)
    if w.dedup:
        layout += 4 * M * E + 4 * R_exp
    s = 1 if w.fp8 else 2
    dispatch = 2 * M * N + R_disp * N * s + (4 * R_disp * (N // 128) if w.fp8 else 0)
    dispatch += 4 * M * (E if w.dedup else k)
    if two_level:
        # partition side: gather the expert rows, write one row per (token, partition);
        # token side: read those rows back, write the token rows
        partial = 2 * R_exp * N + 2 * R_disp * N + 8 * M * k + 4 * R_exp
        reduce = 2 * R_disp * N + 2 * M * N + 4 * M * E
        return {"layout": layout, "dispatch": dispatch, "combine_partial": partial,
                "combine_reduce": reduce}
    combine = 2 * R_exp * N + 2 * M * N + 8 * M * k
    return {"layout": layout, "dispatch": dispatch, "combine": combine}


def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def source_digest(names) -> str:
    """First 16 hex digits of the SHA-256 of the kernel sources ``names``
    (files of the library's csrc/) with comments and whitespace removed, so
    that only a change of the code itself changes it."""
    h = hashlib.sha256()
    for n in names:
        with open(os.path.join(ROOT, "combine_moe_layout_08_b200", "csrc", n)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
        text = re.sub(r"//[^\n]*", "", text)
        h.update(re.sub(r"\s+", "", text).encode())
    return h.hexdigest()[:16]


def traffic_record(kernel: str, workload: str):
    """DRAM bytes per launch from a committed ncu summary, if the kernel's
    code is unchanged since the capture (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    try:
        with open(p) as f:
            rec = json.load(f)[f"{kernel}@{workload}"]
        ok = source_digest(rec["sources"]) == rec["source_sha256_16"]
    except Exception:
        return None
    return float(rec["bytes_per_launch"]) if ok else None


# ---------------------------------------------------------------------------
# clocks during the timed region (NVML polled from a thread; read-only)
# ---------------------------------------------------------------------------
REASONS = {0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
           0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
           0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
           0x100: "display_clock_setting"}


class ClockSampler:
    def __init__(self, torch_device, period_s=0.005):
        self.samples, self.reasons = [], 0
        self.period = period_s
        self._stop = threading.Event()
        self.ok = False
        try:
            import pynvml
            pynvml.nvmlInit()
            self.nv = pynvml
            import torch
            uuid = str(torch.cuda.get_device_properties(torch_device).uuid)
            try:
                self.h = pynvml.nvmlDeviceGetHandleByUUID(("GPU-" + uuid) if not uuid.startswith("GPU-") else uuid)
            except Exception:
                self.h = pynvml.nvmlDeviceGetHandleByIndex(torch_device.index or 0)
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # pragma: no cover - no NVML
            self.err = str(e)

    def _run(self):
        nv = self.nv
        get_r = getattr(nv, "nvmlDeviceGetCurrentClocksEventReasons", None) or \
            nv.nvmlDeviceGetCurrentClocksThrottleReasons
        while not self._stop.is_set():
            try:
                self.samples.append(nv.nvmlDeviceGetClockInfo(self.h, nv.NVML_CLOCK_SM))
                self.reasons |= int(get_r(self.h))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "samples": len(self.samples),
                "reasons": [n for b, n in REASONS.items() if self.reasons & b and b != 0x1]}


# ---------------------------------------------------------------------------
# CPU oracle timing (the reference arm and the cpu_baseline leg)
# ---------------------------------------------------------------------------
def oracle_step_seconds(w, idx, po, gates, x_bits, y_bits, stages=None):
    """One oracle pass (layout, dispatch, combine); returns its seconds and
    the layout, and adds each stage's seconds to ``stages`` if given."""
    import oracle
    t0 = time.perf_counter()
    lay = oracle.layout(idx, po, w.G, w.E_part, w.dedup)
    t1 = time.perf_counter()
    oracle.dispatch(x_bits, lay["disp_token"], w.fp8)
    t2 = time.perf_counter()
    oracle.combine(y_bits, gates, lay["exp_row"])
    t3 = time.perf_counter()
    if stages is not None:
        for k, v in (("layout", t1 - t0), ("dispatch", t2 - t1), ("combine", t3 - t2)):
            stages[k] = stages.get(k, 0.0) + v
    return t3 - t0, lay


def sample_workload(w: W.Workload, tokens: int):
    """The first ``tokens`` tokens of the workload's batch, all inputs drawn
    by the same generators (host copies)."""
    import oracle
    import torch
    d = W.make_inputs(w, device="cpu", with_y=False)
    ws = w.replace(M=tokens)
    idx = d["topk_idx"][:tokens]
    gates = d["topk_weights"][:tokens]
    x_bits = oracle.bf16_bits(d["x"][:tokens])
    y = W.make_expert_outputs(ws)
    return ws, idx, d["part_of"], gates, x_bits, oracle.bf16_bits(y)


def run_reference(args, w):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    tokens = min(w.M, 512)
    ws, idx, po, gates, x_bits, y_bits = sample_workload(w, tokens)
    for _ in range(args.warmup):
        oracle_step_seconds(ws, idx, po, gates, x_bits, y_bits)
    times = []
    lay = None
    for _ in range(args.steps):
        t, lay = oracle_step_seconds(ws, idx, po, gates, x_bits, y_bits)
        times.append(t)
    total = sum(times)
    b = algorithmic_bytes(ws, lay["R_exp"], lay["R_disp"])
    step_bytes = sum(b.values())
    value = step_bytes * args.steps / total / 1e9
    sample = f"first {tokens} of {w.M} tokens of {w.name}, full N/G/topk/E_part, one oracle pass per step"
    line = {
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "GB/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(1e3 * total / args.steps, 3), "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f8e4m3+bf16" if w.fp8 else "bf16",
        "data": "synthetic",
        "tokens_per_s": round(tokens * args.steps / total, 1),
        "config": config_of(w, extra={"sample_tokens": tokens}),
        "cpu_baseline": {"value": round(value, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 4), "unit": "GB/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


METRIC = "dispatch+combine HBM GB/s and tokens/s vs ~8 TB/s roofline at 1 B200"


def replica_workload(w: W.Workload, rank: int) -> W.Workload:
    """Each data-parallel replica draws its own batch of the same shape."""
    return w.replace(seed=w.seed + rank)


def reduce_over_ranks(times, units, device):
    """Max of ``times`` and sum of ``units`` over the ranks of the default
    process group (identity without one)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor(times, dtype=torch.float64, device=device)
    u = torch.tensor(units, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
        dist.all_reduce(u, op=dist.ReduceOp.SUM)
    return t.tolist(), u.tolist()


def config_of(w, extra=None):
    c = {"workload": w.name, "M": w.M, "N": w.N, "G": w.G, "topk": w.topk, "E_part": w.E_part,
         "routing": w.routing, "placement": w.placement, "dedup": w.dedup, "fp8": w.fp8,
         "seed": w.seed, "parallelism": "replicas (one batch per GPU, no collective)"}
    if extra:
        c.update(extra)
    return c


# ---------------------------------------------------------------------------
# our arm
# ---------------------------------------------------------------------------
def graph_kernel_nodes(graph) -> int:
    """Kernel nodes of a captured (not yet instantiated) step graph: the
    launches of this library's kernels per step (the graph holds nothing
    else but event records)."""
    from cuda.bindings import runtime as rt
    raw = graph.raw_cuda_graph()
    err, _, n = rt.cudaGraphGetNodes(raw, 0)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    err, nodes, n = rt.cudaGraphGetNodes(raw, n)
    if err != rt.cudaError_t.cudaSuccess:
        raise RuntimeError(f"cudaGraphGetNodes: {err}")
    kernels = 0
    for node in nodes[:n]:
        err, kind = rt.cudaGraphNodeGetType(node)
        if err != rt.cudaError_t.cudaSuccess:
            raise RuntimeError(f"cudaGraphNodeGetType: {err}")
        kernels += kind == rt.cudaGraphNodeType.cudaGraphNodeTypeKernel
    return kernels


def between_flushes(fns, flush, stream, steps, R=20):
    """Device time of `fns` per repetition, without event nodes inside it:
    one graph of R x [flush, fns] minus one of R x [flush], each replay timed
    whole by events on the stream around it; medians over max(10, steps/10)."""
    import torch
    g_work, g_flush = torch.cuda.CUDAGraph(), torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_work, stream=stream):
        for _ in range(R):
            flush()
            for fn in fns:
                fn()
    with torch.cuda.graph(g_flush, stream=stream):
        for _ in range(R):
            flush()

    def whole(gr, n=max(10, steps // 10)):
        ts = []
        for i in range(n + 3):
            e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
            with torch.cuda.stream(stream):
                e0.record()
                gr.replay()
                e1.record()
            e1.synchronize()
            if i >= 3:
                ts.append(e0.elapsed_time(e1) * 1e3)
        return float(np.median(ts))

    us = (whole(g_work) - whole(g_flush)) / R
    g_work.reset()
    g_flush.reset()
    return us


def run_ours(args, w):
    import torch
    import torch.distributed as dist

    import combine_moe_layout_08_b200 as moe

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world != args.gpus:
        raise SystemExit(f"--gpus {args.gpus} but WORLD_SIZE={world}: launch N>1 with torchrun")
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=180), device_id=dev)

    wr = replica_workload(w, rank)
    d = W.make_inputs(wr, device=dev)
    prob = moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)
    buf = moe.MoEBuffers(prob, dev)
    idx_h, po_h, g_h = d["topk_idx"], d["part_of"], d["topk_weights"]
    idx = torch.from_numpy(idx_h).to(dev)
    po = torch.from_numpy(po_h).to(dev)
    gates = torch.from_numpy(g_h).to(dev)
    x, y = d["x"], d["y"]
    stream = torch.cuda.Stream(dev)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    two_level = args.combine == "two-level"
    if two_level and not w.dedup:
        raise SystemExit("--combine two-level needs a dedup workload")
    separate = args.schedule == "separate"
    fused = not separate and moe.moe_layout_dispatch_fused(prob)
    bm = args.tiles or None
    # eager warm-up through the public API, then one graph per step with
    # external events between the kernels
    with torch.cuda.stream(stream):
        for _ in range(3):
            buf.step(idx, po, x, y, gates, two_level=two_level, separate=separate, block_m=bm)
    stream.synchronize()
    # the step's parts in launch order.  The grouped-GEMM tile metadata, when
    # asked for, comes out of moe_layout_dispatch's own kernels (one part,
    # whatever the schedule), or with --schedule separate from its own
    # kernel after the dispatch.
    if bm and not separate:
        parts = [("layout+dispatch", lambda: buf.layout_dispatch_(idx, po, x, block_m=bm))]
    elif fused:
        parts = [("layout+dispatch", lambda: buf.layout_dispatch_(idx, po, x))]
    else:
        parts = [("layout", lambda: buf.layout_(idx, po)), ("dispatch", lambda: buf.dispatch_(x))]
    if bm and separate:
        parts.append(("tiles", lambda: buf.expert_tiles_(po, bm)))
    # the two-level combine is two kernels: one interval covers the pair
    parts.append(("combine", (lambda: buf.combine_two_level_(y, gates)) if two_level else
                  (lambda: buf.combine_(y, gates))))

    # Two graphs of the same step.  The timed one has events only at its two
    # ends, so consecutive kernels keep their programmatic (early-launch)
    # edges as in production; the second has events between the parts for
    # the per-kernel breakdown (an event node between two kernels replaces
    # that edge with a full dependency, so its parts add up to a little more
    # than the step).
    def capture(inner):
        ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(len(parts) + 1)]
        graph = torch.cuda.CUDAGraph(keep_graph=True)
        with torch.cuda.graph(graph, stream=stream):
            ev[0].record()
            for i, (_, fn) in enumerate(parts):
                fn()
                if inner or i == len(parts) - 1:
                    ev[i + 1].record()
        n = graph_kernel_nodes(graph)
        graph.instantiate()
        return graph, ev, n

    graph, ev, launches_per_step = capture(inner=False)
    pgraph, pev, _ = capture(inner=True)
    R_exp = int(buf.layout.expert_offset[w.G].item())
    R_disp = int(buf.layout.part_offset[w.E_part].item())
    status = int(buf.layout.status.item())
    if status:
        raise SystemExit(f"layout status {status}")
    ab = algorithmic_bytes(wr, R_exp, R_disp, two_level)
    if two_level:
        ab["combine"] = ab.pop("combine_partial") + ab.pop("combine_reduce")
    if bm:
        n_tiles = int(buf.tiles.tile_first[w.G].item())
        ab["tiles"] = 4 * (3 * w.G + w.G + 1) + 12 * n_tiles
    if parts[0][0] == "layout+dispatch":
        ab["layout+dispatch"] = ab.pop("layout") + ab.pop("dispatch") + \
            (ab.pop("tiles") if bm and not separate else 0)
    abytes = {name: ab[name] for name, _ in parts}
    step_bytes = sum(abytes.values())
    move = parts[0][0] if parts[0][0] == "layout+dispatch" else "dispatch"

    def timed_step():
        with torch.cuda.stream(stream):
            flush()
            graph.replay()
        stream.synchronize()
        return ev[0].elapsed_time(ev[-1])

    def parts_step():
        with torch.cuda.stream(stream):
            flush()
            pgraph.replay()
        stream.synchronize()
        return [pev[i].elapsed_time(pev[i + 1]) for i in range(len(parts))]

    # NVTX ranges name the phases for a system-level profiler
    nvtx = torch.cuda.nvtx.range
    with nvtx("warm-up"):
        for _ in range(max(args.warmup, 3)):
            timed_step()
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    step_ms = []
    with ClockSampler(dev) as clk, nvtx("timed steps"):
        for _ in range(args.steps):
            step_ms.append(timed_step())
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    total_ms = float(np.sum(step_ms))
    step_us = np.array(step_ms) * 1e3
    # per-kernel breakdown (untimed for the headline; same flush, same inputs)
    with nvtx("per-kernel breakdown"):
        for _ in range(3):
            parts_step()
        per = np.array([parts_step() for _ in range(args.steps)])   # [K, parts] ms
    kern_ms = {name: float(per[:, i].mean()) for i, (name, _) in enumerate(parts)}
    # the step, and its first part alone, without event nodes inside the
    # work: R x [flush, work] minus R x [flush], each graph timed as a whole
    with nvtx("between flushes"):
        between = {"step": between_flushes([fn for _, fn in parts], flush, stream, args.steps),
                   parts[0][0]: between_flushes([parts[0][1]], flush, stream, args.steps)}

    # end to end through the public API with host buffers
    with nvtx("end to end"):
        e2e = run_e2e(args, wr, buf, idx_h, po_h, g_h, x, y, stream, dev, step_bytes,
                      two_level, separate, bm)

    # aggregate over ranks: bytes and tokens summed, time = max
    (max_ms, max_e2e_ms), (all_bytes, all_tokens, all_e2e_bytes) = reduce_over_ranks(
        [total_ms, e2e["total_ms"]], [step_bytes * args.steps, w.M * args.steps, e2e["bytes"]], dev)

    line = None
    if rank == 0:
        peak, peak_kind = measured_peak()
        dom = max((move, "combine"), key=lambda k: kern_ms[k])
        ach = abytes[dom] / (kern_ms[dom] * 1e-3) / 1e9
        kern_names = {"dispatch": "dispatch_fp8_kernel" if w.fp8 else "dispatch_bf16_kernel",
                      "layout+dispatch": "layout_dispatch_kernel" if fused else
                      "layout kernels+" + ("dispatch_fp8_kernel" if w.fp8 else "dispatch_bf16_kernel"),
                      "tiles": "expert_tiles_kernel",
                      "combine": "combine_partial_kernel+combine_reduce_kernel" if two_level
                      else "combine_kernel"}
        line = {
            "metric": METRIC, "value": round(all_bytes / (max_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(max_ms / args.steps, 5), "higher_is_better": True,
            "step_us": {"mean": round(float(step_us.mean()), 2),
                        "median": round(float(np.median(step_us)), 2),
                        "best": round(float(step_us.min()), 2), "note": "rank 0"},
            "scaling": "weak", "vs_baseline": None, "dtype": "f8e4m3+bf16" if w.fp8 else "bf16",
            "data": "synthetic",
            "tokens_per_s": round(all_tokens / (max_ms * 1e-3), 1),
            "config": config_of(w, extra={
                "R_exp": R_exp, "R_disp": R_disp,
                "combine": "two-level (per partition, then per token)" if two_level else "one-level",
                "schedule": "one kernel for layout + dispatch" if fused and not separate else
                            "separate layout and dispatch kernels",
                "tiles_block_m": bm,
                "l2": "flushed between timed steps (256 MiB write + 256 MiB read, untimed)",
                "timing": "one CUDA graph replay per step; CUDA events recorded inside the graph "
                          "on the launch stream at its start and end"}),
            "kernels_us": {k: round(v * 1e3, 2) for k, v in kern_ms.items()},
            "kernels_note": "per-kernel times from a second graph of the step with events "
                            "between its kernels (mean over the same number of steps)",
            "kernels_gbs": {k: round(abytes[k] / (kern_ms[k] * 1e-3) / 1e9, 1) for k in kern_ms},
            "between_flushes_us": {k: round(v, 2) for k, v in between.items()},
            "between_flushes_note": "one graph of 20 [flush, work] pairs minus one of 20 flushes, "
                                    "each timed whole with events outside it, divided by 20 "
                                    "(median of steps/10 replays): no event node inside the work",
            "algorithmic_bytes_per_step": abytes,
            "roofline": {"bound": "hbm", "kernel": kern_names[dom], "achieved": round(ach, 1),
                         "peak": peak, "unit": "GB/s", "frac": round(ach / peak, 4),
                         "peak_kind": f"of {peak_kind}",
                         "traffic": traffic_record(kern_names[dom], w.name)},
            "frac_of_8tbs": {k: round(abytes[k] / (kern_ms[k] * 1e-3) / 8e12, 4) for k in
                             (move, "combine")},
            "e2e": {"value": round(all_e2e_bytes / (max_e2e_ms * 1e-3) / 1e9, 2), "unit": "GB/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"],
                    "method": "public API, pinned host inputs and output; two buffer sets so "
                              "step i+1's host->device copies overlap step i's kernels and "
                              "device->host copy; timed first copy to last copy",
                    "tokens_per_s": round(w.M * world * args.steps / (max_e2e_ms * 1e-3), 1),
                    "ms_per_step": round(max_e2e_ms / args.steps, 4),
                    "steps": e2e["steps"]},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
        }
    graph.reset()
    pgraph.reset()
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(wr, buf, idx_h, po_h, g_h, x, y)
        line["cpu_baseline_all_cores"] = cpu_baseline_parallel(wr, idx_h, po_h, g_h, x, y)
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def run_e2e(args, w, buf, idx_h, po_h, g_h, x, y, stream, dev, step_bytes,
            two_level=False, separate=False, block_m=None):
    """Public-API calls on host inputs, as a caller streams batches: every
    step copies all of its inputs from pinned host memory to the device, runs
    layout -> dispatch -> combine and copies the output back to pinned host
    memory.  Two buffer sets and three streams (host->device copies, kernels,
    device->host copies) let step i+1's input copies overlap step i's kernels
    and output copy.  The time runs from the first copy's start to the last
    copy's end, so every step's copies are inside it (pipeline fill and drain
    included); the inputs (529 MB at M4096) are larger than L2."""
    import torch

    import combine_moe_layout_08_b200 as moe
    hin = dict(idx=torch.from_numpy(idx_h).pin_memory(), po=torch.from_numpy(po_h).pin_memory(),
               g=torch.from_numpy(g_h).pin_memory(), x=x.cpu().pin_memory(), y=y.cpu().pin_memory())
    sets = [buf, moe.MoEBuffers(buf.prob, dev)]
    din = [{k: torch.empty_like(v, device=dev) for k, v in hin.items()} for _ in sets]
    hout = [torch.empty(buf.out.shape, dtype=buf.out.dtype).pin_memory() for _ in sets]
    h2d = sum(t.numel() * t.element_size() for t in hin.values())
    d2h = hout[0].numel() * hout[0].element_size()
    s_in, s_run, s_out = torch.cuda.Stream(dev), stream, torch.cuda.Stream(dev)

    def pipeline(n):
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        done_in, done_run, done_out = [], [], []
        s_in.wait_stream(torch.cuda.current_stream(dev))
        start.record(s_in)
        for i in range(n):
            b = i % 2
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(done_run[i - 2])    # step i-2 has consumed set b's inputs
                for k, v in hin.items():
                    din[b][k].copy_(v, non_blocking=True)
                done_in.append(torch.cuda.Event())
                done_in[i].record(s_in)
            with torch.cuda.stream(s_run):
                s_run.wait_event(done_in[i])
                if i >= 2:
                    s_run.wait_event(done_out[i - 2])   # set b's output has been read back
                d = din[b]
                out = sets[b].step(d["idx"], d["po"], d["x"], d["y"], d["g"], two_level=two_level,
                                   separate=separate, block_m=block_m)
                done_run.append(torch.cuda.Event())
                done_run[i].record(s_run)
            with torch.cuda.stream(s_out):
                s_out.wait_event(done_run[i])
                hout[b].copy_(out, non_blocking=True)
                done_out.append(torch.cuda.Event())
                done_out[i].record(s_out)
        end.record(s_out)
        end.synchronize()
        return start.elapsed_time(end)

    steps = max(3, min(args.steps, 50))
    pipeline(2)                                         # warm-up
    total = pipeline(steps)
    last = (steps - 1) % 2
    if not torch.equal(hout[last], sets[last].out.cpu()):
        raise SystemExit("end-to-end output mismatch")
    return {"total_ms": total * args.steps / steps, "bytes": step_bytes * args.steps,
            "h2d": h2d, "d2h": d2h, "steps": steps}


def cpu_baseline(w, buf, idx_h, po_h, g_h, x, y, budget_s=10.0):
    """The oracle as it stands, single-threaded, repeated until about
    ``budget_s`` seconds of CPU work: on the whole problem when one pass fits
    the budget, else on its first m tokens (m sized from a timed pass over
    the first 256 tokens so that one pass takes about the budget), with the
    first m*topk expert-row outputs as their y."""
    import oracle
    m = w.M
    probe = min(w.M, 256)
    if probe < w.M:
        t_probe, _ = oracle_step_seconds(w.replace(M=probe), idx_h[:probe], po_h, g_h[:probe],
                                         oracle.bf16_bits(x[:probe]),
                                         oracle.bf16_bits(y[:probe * w.topk]))
        if t_probe * w.M / probe > budget_s:
            m = max(probe, min(w.M, int(probe * budget_s / max(t_probe, 1e-9))))
    ws = w.replace(M=m)
    xb = oracle.bf16_bits(x[:m])
    yb = oracle.bf16_bits(y[:m * w.topk])
    times, stages = [], {}
    lay = None
    while sum(times) < budget_s and len(times) < 50:
        t, lay = oracle_step_seconds(ws, idx_h[:m], po_h, g_h[:m], xb, yb, stages)
        times.append(t)
    b = sum(algorithmic_bytes(ws, lay["R_exp"], lay["R_disp"]).values())
    mean = sum(times) / len(times)
    stage_ms = {k: round(v / len(times) * 1e3, 3) for k, v in stages.items()}
    what = f"full {w.name} problem (M={w.M})" if m == w.M else \
        f"first {m} of the {w.M} tokens of {w.name}"
    model, cores = host_cpu()
    return {"value": round(b / mean / 1e9, 4), "unit": "GB/s", "cores": 1, "kind": "oracle",
            "tokens_per_s": round(m / mean, 1), "cpu": model, "host_cores": cores,
            "ms_per_pass": stage_ms,
            "sample": f"{what}, {len(times)} oracle passes, {sum(times):.1f} s, single thread"}


def host_cpu():
    """Model name and usable cores of this host."""
    model = "unknown"
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    model = line.split(":", 1)[1].strip()
                    break
    except OSError:
        pass
    return model, len(os.sched_getaffinity(0))


def _oracle_shard(job):
    """Worker of cpu_baseline_parallel (its own process): the oracle as it
    stands on one shard of tokens, as a problem of its own, repeated for
    about ``budget`` seconds; returns (seconds, passes, algorithmic bytes)."""
    import oracle
    fields, idx, po, gates, xb, yb, budget = job
    w = W.Workload(**fields)
    times, lay = [], None
    while sum(times) < budget and len(times) < 50:
        t, lay = oracle_step_seconds(w, idx, po, gates, xb, yb)
        times.append(t)
    return sum(times), len(times), sum(algorithmic_bytes(w, lay["R_exp"], lay["R_disp"]).values())


def cpu_baseline_parallel(w, idx_h, po_h, g_h, x, y, budget_s=10.0):
    """The same oracle on every usable host core: one spawned process per
    core, each on its own shard of the first tokens of the batch (the shards
    are independent problems, like data-parallel replicas).  Throughput =
    the shards' bytes / the slowest shard's time.  Returns the reason
    instead if the pool cannot run here."""
    import dataclasses
    import multiprocessing as mp

    import oracle
    model, cores = host_cpu()
    P = max(1, min(cores, 64))
    per = max(1, min(w.M // P, 1024))
    m = per * P
    fields = {f.name: getattr(w, f.name) for f in dataclasses.fields(w)}
    fields["M"] = per
    jobs = []
    for i in range(P):
        t0, t1 = i * per, (i + 1) * per
        jobs.append((fields, idx_h[t0:t1], po_h, g_h[t0:t1], oracle.bf16_bits(x[t0:t1]),
                     oracle.bf16_bits(y[t0 * w.topk:t1 * w.topk]), budget_s))
    # a broken worker (e.g. one that cannot start) raises here instead of
    # hanging, and every result is bounded in time
    from concurrent.futures import ProcessPoolExecutor
    try:
        with ProcessPoolExecutor(P, mp_context=mp.get_context("spawn")) as ex:
            futs = [ex.submit(_oracle_shard, j) for j in jobs]
            res = [f.result(timeout=6 * budget_s + 300) for f in futs]
    except Exception as e:  # a host that cannot run the workers: say so in the line
        return {"unavailable": f"{type(e).__name__}: {e}"}
    slowest = max(r[0] / r[1] for r in res)         # seconds per pass of the slowest shard
    b = sum(r[2] for r in res)
    return {"value": round(b / slowest / 1e9, 4), "unit": "GB/s", "cores": P, "kind": "oracle",
            "tokens_per_s": round(m / slowest, 1), "cpu": model, "host_cores": cores,
            "sample": f"first {m} tokens of {w.name} in {P} shards of {per} (one process "
                      f"per core, each about {budget_s:.0f} s)"}


def run_latency_sweep(args):
    """Decode latency against M on one GPU, in the shape of the Triton-
    distributed issue #117 table (N = 7168, G = 256, topk = 8, bf16,
    M = 2..512): median device time of layout + dispatch (one call, and the
    separate calls) and of combine, L2 flushed before each step (the
    contract line's flush: 256 MiB written, then 256 MiB read).  Prints one
    JSON line; context for the decode path, not the contract line.  Event
    timestamps on this part advance in steps of about 2 us, so single
    intervals of a few us are coarse; medians over many steps are reported.
    step_us comes from a graph with events only at its ends; the parts from
    a graph with an event between them."""
    import dataclasses

    import torch

    import combine_moe_layout_08_b200 as moe

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    base = W.get("decode-M128-uniform")
    stream = torch.cuda.Stream(dev)
    # the contract line's flush: write then read 256 MiB, so each step starts
    # with L2 holding clean lines only (no write-backs charged to the step)
    flush_w = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    flush_r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)
    flush_sink = torch.empty((), dtype=torch.float32, device=dev)

    def flush():
        flush_w.zero_()
        torch.sum(flush_r, dim=0, out=flush_sink)

    rows = []
    for M in SWEEP_M:
        w = dataclasses.replace(base, name=f"decode-M{M}-uniform", M=M)
        d = W.make_inputs(w, device=dev)
        prob = moe.MoEProblem(w.M, w.N, w.G, w.topk, w.E_part, w.dedup, w.fp8)
        idx = torch.from_numpy(d["topk_idx"]).to(dev)
        po = torch.from_numpy(d["part_of"]).to(dev)
        gates = torch.from_numpy(d["topk_weights"]).to(dev)
        row = {"M": M, "one_kernel": moe.moe_layout_dispatch_fused(prob)}
        for separate in (False, True):
            buf = moe.MoEBuffers(prob, dev)
            with torch.cuda.stream(stream):
                buf.step(idx, po, d["x"], d["y"], gates, separate=separate)
            stream.synchronize()
            med = []
            for inner in (False, True):  # the whole step, then its two parts
                ev = [torch.cuda.Event(enable_timing=True, external=True) for _ in range(3)]
                graph = torch.cuda.CUDAGraph()
                with torch.cuda.graph(graph, stream=stream):
                    ev[0].record()
                    if separate:
                        buf.layout_(idx, po)
                        buf.dispatch_(d["x"])
                    else:
                        buf.layout_dispatch_(idx, po, d["x"])
                    if inner:
                        ev[1].record()
                    buf.combine_(d["y"], gates)
                    ev[2].record()
                t = []
                for i in range(max(args.warmup, 3) + args.steps):
                    with torch.cuda.stream(stream):
                        flush()
                        graph.replay()
                    stream.synchronize()
                    if i >= max(args.warmup, 3):
                        t.append((ev[0].elapsed_time(ev[2]),) + ((ev[0].elapsed_time(ev[1]),
                                                                  ev[1].elapsed_time(ev[2]))
                                                                 if inner else (0.0, 0.0)))
                med.append(np.median(np.array(t), axis=0) * 1e3)
                graph.reset()
            # the same step without event nodes inside the graph
            if separate:
                work = [lambda: buf.layout_(idx, po), lambda: buf.dispatch_(d["x"])]
            else:
                work = [lambda: buf.layout_dispatch_(idx, po, d["x"])]
            diff = between_flushes(work + [lambda: buf.combine_(d["y"], gates)], flush, stream,
                                   args.steps)
            # the step alone in a graph, events recorded on the stream around
            # its replay (after the flush), not inside the graph
            g_one = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g_one, stream=stream):
                if separate:
                    buf.layout_(idx, po)
                    buf.dispatch_(d["x"])
                else:
                    buf.layout_dispatch_(idx, po, d["x"])
                buf.combine_(d["y"], gates)
            outer = []
            for i in range(max(args.warmup, 3) + args.steps):
                e0, e1 = (torch.cuda.Event(enable_timing=True) for _ in range(2))
                with torch.cuda.stream(stream):
                    flush()
                    e0.record()
                    g_one.replay()
                    e1.record()
                e1.synchronize()
                if i >= max(args.warmup, 3):
                    outer.append(e0.elapsed_time(e1) * 1e3)
            g_one.reset()
            key = "separate_" if separate else ""
            row[key + "step_us_outer_events"] = round(float(np.median(outer)), 2)
            row[key + "step_us_between_flushes"] = round(diff, 2)
            row[key + "step_us"] = round(float(med[0][0]), 2)
            row[key + "layout_dispatch_us"] = round(float(med[1][1]), 2)
            if not separate:
                row["combine_us"] = round(float(med[1][2]), 2)
        rows.append(row)
    print(json.dumps({"metric": "decode latency against M (us, median, L2 flushed)",
                      "note": "step_us: median of one graph replay with events at its ends; "
                              "step_us_outer_events: median, events recorded on the stream "
                              "around the replay of a graph holding only the step; "
                              "step_us_between_flushes: the step's share of R back-to-back "
                              "[flush, step] replays (no event node inside the graph)",
                      "config": {"N": base.N, "G": base.G, "topk": base.topk,
                                 "E_part": base.E_part, "routing": base.routing},
                      "steps": args.steps, "rows": rows}), flush=True)
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__.split("\n\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", choices=("ours", "reference"), default="ours")
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(W.WORKLOADS))
    ap.add_argument("--tokens", type=int, default=0, metavar="M",
                    help="run the workload's recipe at M tokens instead (a smaller case of the "
                         "same kernels, e.g. for a profiler capture); named NAME@M<M>")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--schedule", choices=("auto", "separate"), default="auto",
                    help="separate: moe_layout + moe_dispatch even where one kernel does both")
    ap.add_argument("--tiles", type=int, default=0, metavar="BM",
                    help="also build the grouped-GEMM tile metadata (tiles of BM rows) each step")
    ap.add_argument("--combine", choices=("one-level", "two-level"), default="one-level",
                    help="two-level: per-partition reduce then per-token sum (dedup workloads)")
    ap.add_argument("--latency-sweep", action="store_true",
                    help="decode latency for M = 2..512 (one JSON line; not the contract line)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        args.warmup = 3
    if args.latency_sweep:
        return run_latency_sweep(args)
    w = W.get(args.workload)
    if args.tokens:
        if args.tokens < 1:
            raise SystemExit("--tokens must be >= 1")
        w = w.replace(name=f"{w.name}@M{args.tokens}", M=args.tokens)
    if args.impl == "reference":
        return run_reference(args, w)
    return run_ours(args, w)


if __name__ == "__main__":
    sys.exit(main())
