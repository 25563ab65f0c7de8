"""Benchmark of the hybrid-head sparse decode-attention step (libychee) on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl lychee|reference]
                    [--workload qwen3_stack_128k|llama3_ragged_stack|qwen3_stack_<N>x<L>]

One step = one decode step of the whole hot path: lychee_decode_stack over all
layers of the workload (per layer: hybrid attention, top-k of the retrieval
heads, combine; the sets chained layer to layer), on seeded synthetic inputs
already resident in HBM.  The default workload is the Qwen3-8B-shaped 36-layer
stack at 128K context (19.3 GB of K/V per step, far larger than L2, so no L2
flush is needed between steps).  The timed steps replay the step captured once
into a CUDA graph; the same steps as direct calls are reported beside them.
Rank 0 prints one JSON line.

Under torchrun (N > 1) every rank runs an independent replica (its own sequence,
seeded by rank); there is no collective on the data path.  Ranks meet at a
barrier around the timed region and the slowest rank's time is reported.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "µs/decode-step & achieved HBM GB/s (% of roofline) at 128K ctx, 1 B200"
UNIT = "µs/decode-step"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ---------------------------------------------------------------- helpers
def measured_peak():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            return float(json.load(f)["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


def max_over_ranks(x, world, device):
    """The largest of the ranks' values (every rank passes its own and gets the
    maximum back); the value itself when there is one rank."""
    if world <= 1:
        return float(x)
    t = torch.tensor([float(x)], device=device, dtype=torch.float64)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def job_us_per_step(ms_per_step_slowest, world):
    """µs per decode step of the whole job: the N replicas each complete one step
    within the slowest rank's step time."""
    return ms_per_step_slowest * 1e3 / world


def attn_traffic_per_launch(alg_bytes_per_launch):
    """DRAM bytes (read + write) of one attention launch: the ncu capture of a
    small case with the same per-layer shape (profiles/attn_kernel.traffic.json)
    gives DRAM bytes per algorithmic byte; a full launch's traffic is that ratio
    times its algorithmic bytes.  None when the kernel sources have changed since
    the capture (the counters no longer describe this kernel)."""
    import hashlib
    try:
        with open(os.path.join(ROOT, "profiles", "attn_kernel.traffic.json")) as f:
            prof = json.load(f)
        h = hashlib.sha256()
        for src in prof["sources"]:
            with open(os.path.join(ROOT, src), "rb") as f:
                h.update(f.read())
        if h.hexdigest() != prof["source_sha256"]:
            return None
        return int(round(prof["traffic_per_algorithmic_byte"] * alg_bytes_per_launch))
    except (OSError, KeyError, ValueError):
        return None


class ClockSampler:
    """Samples SM clock, max clock, power and throttle reasons through NVML while
    running (reads only; changes no setting)."""
    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index, period_s=0.01):
        self.period = period_s
        self.samples = []
        self.max_mhz = None
        self.ok = False
        self._stop = threading.Event()
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = str(torch.cuda.get_device_properties(device_index).uuid)
            handle = None
            for i in range(pynvml.nvmlDeviceGetCount()):
                h = pynvml.nvmlDeviceGetHandleByIndex(i)
                u = pynvml.nvmlDeviceGetUUID(h)
                u = u.decode() if isinstance(u, bytes) else u
                if u.replace("GPU-", "") == uuid.replace("GPU-", ""):
                    handle = h
            if handle is None:
                handle = pynvml.nvmlDeviceGetHandleByIndex(device_index)
            self.nv, self.h = pynvml, handle
            self.max_mhz = float(pynvml.nvmlDeviceGetMaxClockInfo(handle, pynvml.NVML_CLOCK_SM))
            self.ok = True
        except Exception as e:  # no NVML: report the absence, do not fail the bench
            self.err = str(e)

    def _run(self):
        nv, h = self.nv, self.h
        while not self._stop.is_set():
            try:
                mhz = nv.nvmlDeviceGetClockInfo(h, nv.NVML_CLOCK_SM)
                try:
                    rs = nv.nvmlDeviceGetCurrentClocksEventReasons(h)
                except Exception:
                    rs = nv.nvmlDeviceGetCurrentClocksThrottleReasons(h)
                pw = nv.nvmlDeviceGetPowerUsage(h) / 1000.0
                self.samples.append((float(mhz), int(rs), pw))
            except Exception:
                pass
            time.sleep(self.period)

    def __enter__(self):
        if self.ok:
            self._t = threading.Thread(target=self._run, daemon=True)
            self._t.start()
        return self

    def __exit__(self, *a):
        if self.ok:
            self._stop.set()
            self._t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvml unavailable"]}
        if not self.samples:
            return {"sm_mhz": None, "sm_max_mhz": self.max_mhz, "reasons": [], "samples": 0}
        mhz = [s[0] for s in self.samples]
        bits = 0
        for s in self.samples:
            bits |= s[1]
        reasons = sorted(n for b, n in self.REASONS.items() if bits & b and n != "gpu_idle")
        return {"sm_mhz": statistics.median(mhz), "sm_max_mhz": self.max_mhz, "reasons": reasons,
                "samples": len(mhz), "power_w_max": max(s[2] for s in self.samples)}


def make_workload(name, device, seed_offset=0):
    from hybrid_head_sparse_decode_b200 import inputs
    if name == "qwen3_stack_128k":
        return inputs.qwen3_stack_128k(device=device, seed=inputs.BASE_SEED + 2 + seed_offset)
    if name == "llama3_ragged_stack":
        return inputs.llama3_ragged_stack(device=device, seed=inputs.BASE_SEED + 3 + seed_offset)
    if name.startswith("qwen3_stack_"):      # qwen3_stack_<N>x<L>, for small profiling cases
        # the 36-layer stack's head mix scaled to L layers: layer 0 all retrieval,
        # 32 retrieval heads spread over the other 35 layers (about one per layer)
        n, l = (int(x) for x in name[len("qwen3_stack_"):].split("x"))
        return inputs.make_stack(l, 1, 32, 8, 128, n, seed=inputs.BASE_SEED + 2 + seed_offset,
                                 device=device, k_frac=0.3, n_planted=64,
                                 n_extra_retrieval=max(1, round(32 * (l - 1) / 35)) if l > 1 else 0)
    raise SystemExit(f"unknown workload {name}")


def describe(name, prob):
    """The config object of a stack workload's bench line."""
    L, B, Hq, Hkv, d, N = prob.shape
    return {"workload": name, "layers": L, "B": B, "Hq": Hq, "Hkv": Hkv, "d": d,
            "N": N, "seqlens": [int(x) for x in prob.seqlens.cpu()], "k": prob.k,
            "retrieval_heads": int(prob.roles.sum()), "layer0": "all retrieval",
            "io_dtype": "bf16", "accumulate": "fp32",
            "precision": "q.K: bf16 products, fp32 sums (tensor cores); softmax fp32; "
                         "P rounded to bf16 for P.V (tensor cores, fp32 sums), the "
                         "normaliser summing the same rounded weights",
            "l2": "no flush: each step reads %.1f GB of K/V (> 126 MB L2)" % (
                2 * L * B * Hkv * N * d * 2 / 1e9)}


def select_name(block):
    return "argsTopK" if block <= 1 else f"blocks of {block}"


def nearest_rank(sorted_xs, q):
    """The q-quantile of a sorted list by the nearest-rank rule."""
    n = len(sorted_xs)
    return sorted_xs[min(n - 1, max(0, math.ceil(q * n) - 1))]


def union_rows(prob, idx_layers):
    """Rows the method must read per layer and group: n_b for a group holding a
    retrieval head, |union of the heads' incoming sets| for a sparse-only group.
    Returns (union_rows_per_layer, literal_rows_per_layer, dense_rows_per_layer)."""
    L, B, Hq, Hkv, d, N = prob.shape
    G = Hq // Hkv
    dev = idx_layers.device
    union, literal, dense = [], [], []
    for l in range(L):
        u = lit = 0
        roles = prob.roles[l]
        for b in range(B):
            n = int(prob.seqlens[b])
            kb = int(prob.meta["kb"][b])
            for g in range(Hkv):
                hs = list(range(g * G, g * G + G))
                if any(int(roles[h]) == 1 for h in hs):
                    u += n
                    lit += n
                else:
                    mark = torch.zeros(n, dtype=torch.bool, device=dev)
                    for h in hs:
                        # the whole set the head was handed: entries before the
                        # first -1 (a block set may hold more than k_b)
                        row = idx_layers[l - 1, b, h].long()
                        mark[row[row >= 0]] = True
                    u += int(mark.sum())
                    lit += kb
        union.append(u)
        literal.append(lit)
        dense.append(Hkv * int(prob.seqlens.sum()))
    return union, literal, dense


# ---------------------------------------------------------------- our arm
def run_lychee(args, rank, world, device):
    from hybrid_head_sparse_decode_b200 import ops
    from hybrid_head_sparse_decode_b200.inputs import StackProblem

    torch.manual_seed(0)
    prob = make_workload(args.workload, device, seed_offset=rank)
    is_stack = isinstance(prob, StackProblem)
    if not is_stack:
        raise SystemExit("the step benchmark needs a stack workload")
    L, B, Hq, Hkv, d, N = prob.shape
    dt = prob.q.dtype
    row_bytes = 2 * d * prob.q.element_size()
    blk = args.block
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N, prob.k, dt, device, block=blk)
    out = torch.empty((L, B, Hq, d), dtype=dt, device=device)
    fin = torch.empty((B, Hq, prob.k), dtype=torch.int32, device=device)
    idx_layers = torch.empty((L, B, Hq, prob.k), dtype=torch.int32, device=device)
    roles = prob.roles

    def step(r=roles, o=out):
        ops.decode_stack(prob.q, prob.k_caches, prob.v_caches, prob.seqlens, r, prob.k,
                         k_per_seq=prob.k_per_seq, out=o, idx_final=fin, workspace=ws,
                         block=blk)

    # untimed pass that also records every layer's sets, to count algorithmic bytes
    ops.decode_stack(prob.q, prob.k_caches, prob.v_caches, prob.seqlens, roles, prob.k,
                     k_per_seq=prob.k_per_seq, out=out, idx_final=fin, idx_layers=idx_layers,
                     workspace=ws, block=blk)
    st, bits = ops.check_device_error(ws)
    if st != 0:
        raise SystemExit(f"device error {st} bits {bits}")
    urows, lrows, drows = union_rows(prob, idx_layers)
    union_bytes = [u * row_bytes for u in urows]
    literal_bytes = [x * row_bytes for x in lrows]
    dense_bytes = [x * row_bytes for x in drows]
    del idx_layers

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()

    def barrier():
        if world > 1:
            torch.distributed.barrier()

    stream = torch.cuda.current_stream()
    # the step captured once into a CUDA graph (the stack's launches, with their
    # programmatic dependencies) and replayed once per decode step
    gstream = torch.cuda.Stream()
    sgraph = torch.cuda.CUDAGraph()
    with torch.cuda.stream(gstream):
        with torch.cuda.graph(sgraph, stream=gstream):
            ops.decode_stack(prob.q, prob.k_caches, prob.v_caches, prob.seqlens, roles, prob.k,
                             k_per_seq=prob.k_per_seq, out=out, idx_final=fin, workspace=ws,
                             block=blk, stream=gstream)
    for _ in range(args.warmup):
        sgraph.replay()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    sampler = ClockSampler(device.index)
    # timed region: the steps alone (the reported value), graph replays
    barrier()
    torch.cuda.synchronize()
    with sampler:
        t0.record(stream)
        for _ in range(args.steps):
            sgraph.replay()
        t1.record(stream)
        torch.cuda.synchronize()
    barrier()
    ms_total = t0.elapsed_time(t1)
    # the same steps as direct calls of the library (host work per call included)
    torch.cuda.synchronize()
    t0.record(stream)
    for _ in range(args.steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    direct_ms = max_over_ranks(t0.elapsed_time(t1), world, device) / args.steps
    # the same steps again with every library launch bracketed by CUDA events on
    # its stream: per-kernel durations for the roofline of the attention kernel
    prof = ops.Profile(max_launches=args.steps * (4 * L + 2) + 16)
    torch.cuda.synchronize()
    with prof:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
    # per-step spread: an event after every replay of another pass of the same steps
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps + 1)]
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(args.steps):
        sgraph.replay()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    del sgraph
    per_step = sorted(ev[i].elapsed_time(ev[i + 1]) for i in range(args.steps))
    ms_total = max_over_ranks(ms_total, world, device)
    ms_step = ms_total / args.steps
    recs = prof.records
    attn = [ms for k, ms in recs if k == "attn"]
    kinds = {}
    for k, ms in recs:
        kinds.setdefault(k, [0, 0.0])
        kinds[k][0] += 1
        kinds[k][1] += ms
    # per-launch algorithmic bytes of the attention kernel, layer by layer
    attn_bytes_per_step = sum(union_bytes)
    attn_ms_per_step = sum(attn) / args.steps if attn else float("nan")   # serialised
    # the attention launches as they run in the step: the library's span mode
    # records one event before each call's first attention launch and one after
    # its last, nothing in between (the layers still overlap); their average
    # duration is the span / L
    sprof = ops.Profile(max_launches=args.steps + 8, spans=True)
    torch.cuda.synchronize()
    with sprof:
        for _ in range(args.steps):
            step()
        torch.cuda.synchronize()
    spans = sorted(ms for k, ms in sprof.records if k == "attn_span")
    span_ms = statistics.median(spans) if spans else float("nan")
    achieved = attn_bytes_per_step / (span_ms * 1e-3) / 1e9
    achieved_serial = attn_bytes_per_step / (attn_ms_per_step * 1e-3) / 1e9
    peak, peak_kind = measured_peak()

    # dense comparator: the same kernels with every head a retrieval head
    dense_roles = torch.ones_like(roles)
    dense_out = torch.empty_like(out)
    for _ in range(max(1, args.warmup // 2)):
        step(dense_roles, dense_out)
    dsteps = max(3, args.steps // 4)
    torch.cuda.synchronize()
    d0, d1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    d0.record(stream)
    for _ in range(dsteps):
        step(dense_roles, dense_out)
    d1.record(stream)
    torch.cuda.synchronize()
    dense_ms = d0.elapsed_time(d1) / dsteps
    # its per-kernel split (events around every launch, which serialise it)
    dprof = ops.Profile(max_launches=dsteps * (4 * L + 2) + 16)
    torch.cuda.synchronize()
    with dprof:
        for _ in range(dsteps):
            step(dense_roles, dense_out)
        torch.cuda.synchronize()
    dkinds = {}
    for k, ms in dprof.records:
        dkinds[k] = dkinds.get(k, 0.0) + ms / dsteps

    # the step before the attention of a decode step, timed on its own: the
    # current token's K/V rows into every layer's cache (the rows already there,
    # so the caches do not change)
    b_idx = torch.arange(B, device=device)
    last = (prob.seqlens.long() - 1)
    k_new = [kc[b_idx, :, last].contiguous() for kc in prob.k_caches]
    v_new = [vc[b_idx, :, last].contiguous() for vc in prob.v_caches]

    def append_all():
        for l in range(L):
            ops.append_kv(k_new[l], v_new[l], prob.k_caches[l], prob.v_caches[l], prob.seqlens)

    for _ in range(2):
        append_all()
    # replayed from a CUDA graph, so that the host's per-call work is not timed
    gstream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    torch.cuda.synchronize()
    with torch.cuda.stream(gstream):
        with torch.cuda.graph(graph, stream=gstream):
            append_all()
    for _ in range(2):
        graph.replay()
    a0, a1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    a0.record(stream)
    for _ in range(args.steps):
        graph.replay()
    a1.record(stream)
    torch.cuda.synchronize()
    append_ms = a0.elapsed_time(a1) / args.steps
    del graph

    # end to end through the public call with host buffers: q (and the per-sequence
    # lengths and budgets) copied in from pinned memory, out and the final sets read
    # back every step.  The K/V caches are the model's resident decode state.
    q_h = prob.q.cpu().pin_memory()
    sl_h = prob.seqlens.cpu().pin_memory()
    kb_h = prob.k_per_seq.cpu().pin_memory()
    out_h = torch.empty(out.shape, dtype=dt).pin_memory()
    fin_h = torch.empty(fin.shape, dtype=torch.int32).pin_memory()
    q_d = torch.empty_like(prob.q)
    sl_d = torch.empty_like(prob.seqlens)
    kb_d = torch.empty_like(prob.k_per_seq)

    def e2e_step():
        q_d.copy_(q_h, non_blocking=True)
        sl_d.copy_(sl_h, non_blocking=True)
        kb_d.copy_(kb_h, non_blocking=True)
        ops.decode_stack(q_d, prob.k_caches, prob.v_caches, sl_d, roles, prob.k, k_per_seq=kb_d,
                         out=out, idx_final=fin, workspace=ws, block=blk)
        out_h.copy_(out, non_blocking=True)
        fin_h.copy_(fin, non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(args.steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    barrier()
    e_ms = e0.elapsed_time(e1)
    e_ms = max_over_ranks(e_ms, world, device)
    h2d = (q_h.numel() * q_h.element_size() + sl_h.numel() * 4 + kb_h.numel() * 4)
    d2h = out_h.numel() * out_h.element_size() + fin_h.numel() * 4

    us_step_job = job_us_per_step(ms_step, world)
    step_gbs = sum(union_bytes) / (ms_step * 1e-3) / 1e9
    result = {
        "metric": METRIC, "value": round(us_step_job, 3), "unit": UNIT, "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 5),
        "higher_is_better": False, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded; planted high-affinity keys)",
        "config": dict(describe(args.workload, prob),
                       select=select_name(blk)),
        "us_per_layer": round(ms_step * 1e3 / L, 3),
        # the attention launches of layer 0 (all retrieval heads) and of the
        # other layers, from the events around every launch (serialised)
        "attn_us_by_layer": {
            "layer0_median": round(statistics.median(attn[0::L]) * 1e3, 2) if attn else None,
            "others_median": round(statistics.median([a for i, a in enumerate(attn) if i % L])
                                   * 1e3, 2) if attn and L > 1 else None},
        "step_ms_spread": {"p10": round(nearest_rank(per_step, 0.1), 5),
                           "median": round(nearest_rank(per_step, 0.5), 5),
                           "p90": round(nearest_rank(per_step, 0.9), 5),
                           "steps": len(per_step), "rank": rank},
        "step_hbm_gbs_union": round(sum(union_bytes) / (ms_step * 1e-3) / 1e9, 1),
        "step_hbm_gbs_literal": round(sum(literal_bytes) / (ms_step * 1e-3) / 1e9, 1),
        "bytes_per_step": {"union": sum(union_bytes), "literal": sum(literal_bytes),
                           "dense": sum(dense_bytes)},
        # the dominant kernel's roofline (attention launches only) ...
        "roofline": {"bound": "hbm", "achieved": round(achieved, 1), "peak": peak,
                     "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": attn_traffic_per_launch(attn_bytes_per_step / L),
                     "algorithmic_bytes_per_launch": int(attn_bytes_per_step / L),
                     "kernel": "attn_kernel (hybrid attention, all layers)",
                     "launch_us": round(span_ms * 1e3 / L, 2),
                     "duration_rule": "CUDA events before a step's first attention launch and "
                                      "after its last (the launches run back to back, the "
                                      "selections overlapping them): span / L, median of "
                                      "%d steps" % len(spans),
                     "serialised": {"launch_us": round(attn_ms_per_step * 1e3 / L, 2),
                                    "frac": round(achieved_serial / peak, 4),
                                    "rule": "events around every launch, which serialise the "
                                            "layers; a launch then also holds the previous "
                                            "layer's combine at its end"},
                     "scope": "attention kernel launches only; the whole step is step_roofline",
                     "peak_source": peak_kind, "frac_of_nominal_8tbs": round(achieved / NOMINAL_HBM_GBS, 4),
                     "bytes_rule": "union rows x 512 B per launch"},
        # ... and the whole decode step's (the figure the 70 % target is set on)
        "step_roofline": {"achieved": round(step_gbs, 1), "peak": peak, "unit": "GB/s",
                          "frac": round(step_gbs / peak, 4),
                          "frac_of_nominal_8tbs": round(step_gbs / NOMINAL_HBM_GBS, 4),
                          "bytes_rule": "union rows x 512 B over every layer / ms_per_step"},
        "kernels_ms_per_step": {k: round(v[1] / args.steps, 4) for k, v in kinds.items()},
        "dense_comparator": {"ms_per_step": round(dense_ms, 4),
                             "hbm_gbs": round(sum(dense_bytes) / (dense_ms * 1e-3) / 1e9, 1),
                             "speedup_hybrid_vs_dense": round(dense_ms / ms_step, 3),
                             "kernels_ms_per_step": {k: round(v, 4) for k, v in dkinds.items()}},
        "e2e": {"value": round(job_us_per_step(e_ms / args.steps, world), 3), "unit": UNIT,
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "timing": "value: the step captured once into a CUDA graph, replayed once per step",
        "direct_call": {"ms_per_step": round(direct_ms, 5),
                        "note": "the same steps as direct calls of lychee_decode_stack"},
        "append_kv": {"ms_per_step": round(append_ms, 4), "launches_per_step": L,
                      "note": "the current token's K/V rows into all layers' caches, one launch "
                              "per layer, replayed from a CUDA graph; the step above starts from "
                              "caches that hold them"},
        "gpu_launches": sum(v[0] for v in kinds.values()),
        "clocks": sampler.summary(),
    }
    return result, prob, union_bytes


# ---------------------------------------------------------------- the one-layer sweep
def layer_rows(prob, all_retrieval):
    """(union rows, literal rows) of one layer: n_b for a KV group holding a
    retrieval head; for a sparse-only group the size of the union of its heads'
    incoming sets (union) or k_b (literal)."""
    B, Hq, Hkv, d, N = prob.shape
    G = Hq // Hkv
    role = prob.role.cpu()
    u = lit = 0
    for b in range(B):
        n = int(prob.seqlens[b])
        kb = int(prob.meta["kb"][b])
        for g in range(Hkv):
            hs = range(g * G, g * G + G)
            if all_retrieval or any(int(role[h]) == 1 for h in hs):
                u += n
                lit += n
                continue
            mark = torch.zeros(n, dtype=torch.bool, device=prob.idx_in.device)
            for h in hs:
                row = prob.idx_in[b, h].long()
                mark[row[row >= 0]] = True
            u += int(mark.sum())
            lit += kb
    return u, lit


def flush_l2(buf):
    """Evict the caches' lines from L2: write a buffer larger than L2, then
    read it back, so that the dirty lines of the write are written back here
    and not during the next timed call."""
    buf.zero_()
    buf.sum()


def time_layer_call(prob, steps, warmup, flush, all_retrieval):
    """CUDA-event times (ms) of the single-layer call, L2 flushed before every
    call, and the attention kernel's own median launch time from the library's
    launch profiler over the same number of calls."""
    from hybrid_head_sparse_decode_b200 import ops
    B, Hq, Hkv, d, N = prob.shape
    dt = prob.q.dtype
    role = torch.ones_like(prob.role) if all_retrieval else prob.role
    idx_in = None if all_retrieval else prob.idx_in
    ws = ops.alloc_workspace(B, Hq, Hkv, d, N, prob.k, dt, prob.q.device)
    out = torch.empty_like(prob.q)
    idx_out = torch.empty((B, Hq, prob.k), dtype=torch.int32, device=prob.q.device)

    def call():
        ops.hybrid_decode_attn(prob.q, prob.k_cache, prob.v_cache, prob.seqlens, role, idx_in,
                               prob.k, k_per_seq=prob.k_per_seq, out=out, idx_out=idx_out,
                               workspace=ws)

    for _ in range(warmup):
        flush_l2(flush)
        call()
    st, bits = ops.check_device_error(ws)
    if st != 0:
        raise SystemExit(f"device error {st} bits {bits}")
    stream = torch.cuda.current_stream()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
          for _ in range(steps)]
    for e0, e1 in ev:
        flush_l2(flush)
        e0.record(stream)
        call()
        e1.record(stream)
    torch.cuda.synchronize()
    per = sorted(e0.elapsed_time(e1) for e0, e1 in ev)
    prof = ops.Profile(max_launches=4 * steps + 8)
    with prof:
        for _ in range(steps):
            flush_l2(flush)
            call()
        torch.cuda.synchronize()
    attn = sorted(ms for k, ms in prof.records if k == "attn")
    split = {}
    for k, ms in prof.records:
        split.setdefault(k, []).append(ms)
    split = {k: round(statistics.median(v) * 1e3, 2) for k, v in split.items()}
    return per, attn, split


def run_sweep(args, device):
    """Every point of the one-layer sweep (Qwen3-8B head layout, 4 retrieval
    heads; N from 4K to 256K at B = 1, B in {4, 16} at 64K; k = 30 % of n_b or
    2048), each also run with every head a retrieval head (the dense twin)."""
    from hybrid_head_sparse_decode_b200 import inputs
    peak, peak_kind = measured_peak()
    flush = torch.empty(64 << 20, dtype=torch.int32, device=device)   # 256 MB > L2
    points = []
    for B, N, km in inputs.sweep_points():
        rec = {"B": B, "N": N, "k": "30%" if km == "frac" else km}
        for mode in ("hybrid", "dense"):
            prob = inputs.sweep_layer(B, N, km, device=device, all_retrieval=False)
            dense = mode == "dense"
            u, lit = layer_rows(prob, dense)
            per, attn, split = time_layer_call(prob, args.steps, args.warmup, flush, dense)
            row_bytes = 2 * prob.shape[3] * prob.q.element_size()
            med = nearest_rank(per, 0.5)
            am = nearest_rank(attn, 0.5) if attn else float("nan")
            rec[mode] = {
                "us": round(med * 1e3, 2), "us_p10": round(nearest_rank(per, 0.1) * 1e3, 2),
                "us_p90": round(nearest_rank(per, 0.9) * 1e3, 2),
                "attn_us": round(am * 1e3, 2),
                "union_bytes": u * row_bytes, "literal_bytes": lit * row_bytes,
                "gbs_union": round(u * row_bytes / (med * 1e-3) / 1e9, 1),
                "gbs_literal": round(lit * row_bytes / (med * 1e-3) / 1e9, 1),
                "attn_gbs_union": round(u * row_bytes / (am * 1e-3) / 1e9, 1),
                "attn_frac": round(u * row_bytes / (am * 1e-3) / 1e9 / peak, 4),
                "kernels_us": split}
            del prob
            torch.cuda.empty_cache()
        rec["speedup_hybrid_vs_dense"] = round(rec["dense"]["us"] / rec["hybrid"]["us"], 3)
        points.append(rec)
        print(json.dumps({"sweep_point": rec}), flush=True)
    return {"metric": "µs per single-layer call and achieved HBM GB/s, one-layer sweep",
            "unit": "µs", "n_gpus": 1, "steps": args.steps, "warmup": args.warmup,
            "higher_is_better": False, "dtype": "bf16", "data": "synthetic (seeded)",
            "config": {"workload": "qwen3_layer_sweep", "Hq": 32, "Hkv": 8, "d": 128,
                       "retrieval_heads": 4, "incoming_sets": "random",
                       "l2": "flushed before every call by writing a 256 MB buffer and reading it back (no dirty lines left to write back during the call)",
                       "timed": "the whole layer call (set bitmaps, attention, top-k + "
                                "combine); attn_* from the attention kernel's own launch"},
            "peak": {"hbm_gbs": peak, "source": peak_kind}, "points": points}


# ---------------------------------------------------------------- the oracle arm
def oracle_chain_time(prob, layers, nthreads, block=0):
    """Time the oracle's own chain over the given leading layers of the stack
    (block > 1: block-granular selection); returns per-layer seconds."""
    import numpy as np

    import oracle

    def bits(t):
        t = t.detach().contiguous().cpu()
        return t.view(torch.int16).numpy().view(np.uint16)

    L, B, Hq, Hkv, d, N = prob.shape
    seqlens = prob.seqlens.cpu().numpy()
    kps = prob.k_per_seq.cpu().numpy()
    idx = np.full((B, Hq, prob.k), -1, np.int32)
    times = []
    for l in range(layers):
        q, K, V = bits(prob.q[l]), bits(prob.k_caches[l]), bits(prob.v_caches[l])
        t = time.perf_counter()
        _, idx, _ = oracle.hybrid_layer(q, K, V, seqlens, prob.roles[l].numpy(), idx, prob.k,
                                        k_per_seq=kps, nthreads=nthreads,
                                        block=max(1, block))
        times.append(time.perf_counter() - t)
    return times


def scale_to_step(times, L):
    """Layer 0 (all retrieval) timed as is; the other layers by the mean of the
    sampled ones."""
    rest = times[1:] if len(times) > 1 else times
    return times[0] + sum(rest) / len(rest) * (L - 1)


def cpu_model():
    """The host CPU's model string (from /proc/cpuinfo), or the platform's."""
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    import platform
    return platform.processor() or platform.machine()


def cpu_baseline(prob, block=0, single_layers=2):
    """The oracle as it stands on the host: (a) its whole chain over every layer
    of the workload, OpenMP over (sequence, head) on all host cores -- one
    measured decode step; (b) single-threaded over the first layers, scaled to
    the step (layer 0 as timed, the mean of the others for the rest)."""
    import oracle
    oracle.build()
    L, B, Hq = prob.shape[0], prob.shape[1], prob.shape[2]
    nthreads = os.cpu_count() or 1
    full = oracle_chain_time(prob, L, nthreads, block)
    one = oracle_chain_time(prob, min(single_layers, L), 1, block)
    cores = min(nthreads, B * Hq)
    return {"value": round(sum(full) * 1e6, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
            "cpu_model": cpu_model(), "nproc": nthreads,
            "single_thread": {"value": round(scale_to_step(one, L) * 1e6, 1), "unit": UNIT,
                              "cores": 1,
                              "sample": f"layers 0..{len(one) - 1} single-threaded "
                                        f"({sum(one):.1f} s), scaled to {L} layers"},
            "sample": f"one whole decode step: the oracle's own chain over all {L} layers of "
                      f"the same workload, OpenMP over (sequence, head) on {cores} threads "
                      f"({sum(full):.1f} s)"}


def run_reference(args, rank, world):
    """The reference arm: the fp64 oracle as it stands, on host cores (OpenMP
    over (sequence, head)), each step its own chain over every layer of the
    workload.  Rank 0 only."""
    if rank != 0:
        return None
    import oracle
    oracle.build()
    device = torch.device("cuda", 0) if torch.cuda.is_available() else torch.device("cpu")
    prob = make_workload(args.workload, device)
    L = prob.shape[0]
    nthreads = os.cpu_count() or 1
    for _ in range(min(args.warmup, 1)):
        oracle_chain_time(prob, 1, nthreads, args.block)
    per = [sum(oracle_chain_time(prob, L, nthreads, args.block)) for _ in range(args.steps)]
    us = statistics.median(per) * 1e6
    B, Hq = prob.shape[1], prob.shape[2]
    cores = min(nthreads, B * Hq)
    cb = {"value": round(us, 1), "unit": UNIT, "cores": cores, "kind": "oracle",
          "cpu_model": cpu_model(), "nproc": nthreads,
          "sample": f"every step the oracle's own chain over all {L} layers (OpenMP over "
                    f"(sequence, head), {cores} threads); median of {args.steps} steps, "
                    f"{sum(per):.1f} s in all"}
    return {"impl": "reference", "metric": METRIC, "value": round(us, 1), "unit": UNIT,
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(us / 1e3, 3), "higher_is_better": False, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic (seeded)",
            "config": dict(describe(args.workload, prob), select=select_name(args.block)),
            "cpu_baseline": cb,
            "e2e": {"value": round(us, 1), "unit": UNIT, "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------- main
def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lychee", choices=["lychee", "reference"])
    ap.add_argument("--workload", default="qwen3_stack_128k")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--sweep", action="store_true",
                    help="time every point of the one-layer sweep and its all-retrieval "
                         "twin instead of the stack step (one JSON line per point, then a "
                         "summary line)")
    ap.add_argument("--block", type=int, default=0,
                    help="0: retrieval heads hand on argsTopK sets (the method's step); "
                         "B > 1: block-granular sets of B positions")
    args = ap.parse_args()
    if args.warmup < 3 and args.impl == "lychee":
        args.warmup = 3

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle runs on host cores, on rank 0 only; other ranks leave at once
        res = run_reference(args, rank, world)
        if res is not None:
            print(json.dumps(res), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300),
                                             device_id=torch.device("cuda", local))

    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    if args.sweep:
        if world > 1:
            raise SystemExit("the sweep runs on one GPU")
        print(json.dumps(run_sweep(args, device)), flush=True)
        return
    res, prob, _ = run_lychee(args, rank, world, device)
    if rank == 0:
        if world == 1 and not args.no_cpu_baseline:
            res["cpu_baseline"] = cpu_baseline(prob, block=args.block)
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
