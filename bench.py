#!/usr/bin/env python
"""Benchmark of the single-GPU MoE dispatch + combine hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
    python -m torch.distributed.run --nproc-per-node N ... bench.py --gpus N

One step = one pass of the whole hot path over one batch:
    dispatch layout (count + look-back scan, emit)  ->  permute bf16  ->
    permute + block FP8  ->  permute + NVFP4  ->  combine (bf16 out)
on the metric workload N=8192 tokens, H=7168, E=256 experts, top_k=8,
S=8 segments, recv_capacity = N*top_k (seeded synthetic inputs, uniform
distinct routing, 1% outlier rows, expert outputs ~N(0,1)).

Each rank runs its own batch (replicas; weak scaling, no data-path
collective); the timed region is bracketed by a barrier and device
synchronisation, every step is timed with CUDA events on the launching stream,
and the max over ranks is reported.  L2 is flushed before every step (a write
of a buffer twice its size, then a read of another such buffer so the dirty
lines are retired there), outside the events.  Rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "dispatch+combine tokens/s and HBM GB/s (% of peak) at N=8192 H=7168 E=256 k=8"
WORKLOAD = "fp8_metric"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0   # B200 HBM3e, nominal (DGX figure)

# dram bytes (read + write) per launch from one ncu capture of the DRAM
# counters on the metric workload (profiles/traffic_fp8_metric.md), keyed by
# kernel; valid only while the kernel's device code is unchanged (sha256
# prefix of its text and the shared helpers at capture time)
NCU_TRAFFIC: dict[str, dict] = {
    "permute_bf16": {"bytes_per_launch": 118010880 + 881758976, "src_sha": "a0218bc31711bbc1"},
    "permute_fp8": {"bytes_per_launch": 118075392 + 422765568, "src_sha": "28d14b0055d493d3"},
    "permute_nvfp4": {"bytes_per_launch": 118034432 + 203461888, "src_sha": "84fc6bc2afa495d1"},
    "combine": {"bytes_per_launch": 940088320 + 64898048, "src_sha": "709371a62977d2c7"},
}


# the kernel function each phase runs: (source file, function name)
KERNEL_SRC = {"permute_bf16": ("permute.cu", "permute_bf16_kernel"),
              "permute_fp8": ("permute.cu", "permute_fp8_kernel"),
              "permute_nvfp4": ("permute.cu", "permute_fp4_kernel"),
              "combine": ("combine.cu", "combine_kernel")}


def _kernel_src_sha(phase: str) -> str:
    """Hash of the device code a phase's ncu counters depend on: its kernel
    function's text (from the __global__ line to the closing brace in column
    0) plus the shared device helpers (common.cuh).  Host-side edits of the
    same file leave it unchanged; any change to the kernel or the helpers
    invalidates the stored traffic."""
    fn, name = KERNEL_SRC[phase]
    csrc = os.path.join(ROOT, "combine_topk_ids_scan_b200", "csrc")
    text = open(os.path.join(csrc, fn)).read()
    at = text.index(f"    {name}(")
    start = text.rindex("__global__", 0, at)
    start = text.rindex("\n", 0, start) + 1
    end = text.index("\n}\n", at) + 3
    h = hashlib.sha256(text[start:end].encode())
    h.update(open(os.path.join(csrc, "common.cuh"), "rb").read())
    return h.hexdigest()[:16]


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            pk = json.load(f)
        return float(pk["hbm_gbs"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, "fallback"


# ------------------------------------------------------------------ bytes
def algorithmic_bytes(w, total_rows: int) -> dict:
    """Compulsory HBM bytes per step phase (each input read once, each output
    written once) for workload w whose layout routed `total_rows` rows."""
    N, H, k, P, rows, E, S = w.N, w.H, w.k, w.P, w.rows, w.E, w.S
    maps_read = 4 * P + 4 * rows          # pair_slot + row_src read by a permute
    return {
        "layout": 4 * P + 4 * P + 4 * rows + P + 8 * E + 4 + 16 * S,
        "permute_bf16": 2 * N * H + maps_read + 2 * rows * H,
        "permute_fp8": 2 * N * H + maps_read + rows * H + 4 * rows * (H // 128),
        "permute_nvfp4": 2 * N * H + maps_read + rows * H // 2 + rows * (H // 16) + 4,
        "combine": 2 * total_rows * H + 4 * P + 4 * P + 2 * N * H,
    }


# ------------------------------------------------------------------ clocks
class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""

    FIELDS = ("uuid,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, uuid: str | None):
        self.uuid = uuid
        self.lines: list[str] = []
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except Exception:
            self.proc = None
            return
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in self.lines:
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            if self.uuid and self.uuid not in f[0]:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
                power.append(float(f[3]))
            except ValueError:
                continue
            for name, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax),
                "power_w_max": max(power), "samples": len(sm), "reasons": sorted(reasons)}


# ------------------------------------------------------------------ dist
def dist_env():
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return rank, world, local


def seed_for_rank(rank: int) -> int | None:
    """Rank 0 runs the canonical seeded batch; every other rank draws its own
    independent batch of the same shape (weak scaling over replicas)."""
    return None if rank == 0 else 1002 + 7919 * rank


def max_over_ranks(values, device, world: int):
    """Element-wise max of a list of floats over all ranks (a timing
    reduction only; the data path has no collective)."""
    if world <= 1:
        return [float(v) for v in values]
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(v) for v in values], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(v) for v in t.tolist()]


# ------------------------------------------------------------------ oracle
def oracle_tokens_per_s(w, n_tokens: int, start: int = 0,
                        threads: int = 1) -> tuple[float, float]:
    """Time the CPU oracle (as it stands) on the sub-batch of tokens
    [start, start+n): its own layout (packed with recv_capacity = n*k, or the
    workload's expert capacity), the permutes the shape allows and the
    combine.  threads > 1 splits the permutes' rows and the combine's tokens
    over a thread pool (each oracle call is single-threaded C and releases
    the GIL; the layout stays one call).  Returns (tokens/s, seconds)."""
    import concurrent.futures as cf

    import oracle
    oracle.build()
    n = min(n_tokens, w.N)
    idx = (np.arange(n) + start) % w.N
    ids = np.ascontiguousarray(w.ids[idx])
    hidden = np.ascontiguousarray(w.hidden[idx])
    gates = np.ascontiguousarray(w.gates[idx])
    if w.expert_capacity > 0:
        lay_kw, rows = dict(expert_capacity=w.expert_capacity), w.E * w.expert_capacity
    else:
        lay_kw, rows = dict(recv_capacity=n * w.k), n * w.k
    X = np.ascontiguousarray(w.expert_out[:rows]) if w.expert_out is not None else None

    def split(fn, m, *arrays):
        if threads <= 1:
            return fn(*arrays)
        step = max(1, -(-m // threads))
        with cf.ThreadPoolExecutor(threads) as ex:
            list(ex.map(lambda i: fn(*[a[i:i + step] for a in arrays]), range(0, m, step)))

    t0 = time.perf_counter()
    lay = oracle.layout(ids, w.E, w.S, w.H, **lay_kw)
    rs = lay.row_src
    split(lambda r: oracle.permute_bf16(hidden, r), rows, rs)
    if w.H % 128 == 0:
        split(lambda r: oracle.permute_fp8(hidden, r), rows, rs)
    if w.H % 32 == 0:
        split(lambda r: oracle.permute_nvfp4(hidden, r, w.global_scale), rows, rs)
    if X is not None:
        split(lambda g, ps: oracle.combine(X, g, ps), n, gates, lay.pair_slot)
    dt = time.perf_counter() - t0
    return n / dt, dt


def run_reference(args, rank: int, world: int) -> int:
    """Reference arm: the CPU oracle timed on bounded samples of the workload."""
    if rank != 0:
        return 0
    from combine_topk_ids_scan_b200.inputs import make_workload
    w = make_workload(WORKLOAD)
    # ~1.8 ms of oracle work per token; keep the whole run near a minute
    per_step = max(8, min(2048, int(60.0 / max(1, args.steps + args.warmup) / 1.8e-3)))
    for i in range(args.warmup):
        oracle_tokens_per_s(w, per_step, start=i * per_step)
    times = []
    for i in range(args.steps):
        _, dt = oracle_tokens_per_s(w, per_step, start=(args.warmup + i) * per_step)
        times.append(dt)
    ms = 1e3 * sum(times) / len(times)
    value = per_step / (ms / 1e3)
    sample = (f"{per_step} consecutive tokens of the {WORKLOAD} batch per step "
              f"(own layout with recv_capacity = {per_step}*k)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp32",
        "data": "synthetic", "config": workload_config(w),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                         "sample": sample, "box_cores": os.cpu_count()},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# every workload of the benchmark set and the oracle sample timed beside it
# (tokens; about a second or two of single-threaded oracle work each)
CONFIG_SET = ("tiny", "mid_zipf", "fp8_metric", "nvfp4_hot", "decode_capacity",
              "balanced_static")
CPU_SAMPLE_TOKENS = {"tiny": 512, "mid_zipf": 512, "fp8_metric": 1024, "nvfp4_hot": 1024,
                     "decode_capacity": 128, "balanced_static": 1024}


def measure_workload(B, torch, w, dev, stream, flush_l2, n_steps: int, peak: float) -> dict:
    """Times one workload of the benchmark set on this GPU (inputs resident,
    L2 flushed before every step, outside the events): the whole step
    (layout, the permutes the shape allows, combine) between two events,
    the dispatch bf16 + combine trio between two events, and each kernel
    with an event between kernels.  Returns a JSON-ready dict."""
    prob = B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity)
    buf = B.Buffers(prob, device=dev)
    d_ids = torch.from_numpy(w.ids).to(dev)
    d_hidden = torch.from_numpy(w.hidden.view(np.int16)).to(dev).view(torch.bfloat16)
    d_gates = torch.from_numpy(w.gates).to(dev)
    d_x = torch.from_numpy(w.expert_out.view(np.int16)).to(dev).view(torch.bfloat16)
    d_gs = torch.tensor([w.global_scale], dtype=torch.float32, device=dev)
    d_y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    calls = {"layout": lambda: B.layout(prob, d_ids, buf),
             "permute_bf16": lambda: B.moe_permute(prob, d_hidden, buf.row_src, buf.pair_slot,
                                                   buf.out)}
    if w.H % 128 == 0:
        calls["permute_fp8"] = lambda: B.moe_permute_quant_fp8(
            prob, d_hidden, buf.row_src, buf.pair_slot, buf.out_fp8, buf.scales_fp8)
    if w.H % 32 == 0:
        calls["permute_nvfp4"] = lambda: B.moe_permute_quant_nvfp4(
            prob, d_hidden, buf.row_src, buf.pair_slot, d_gs, buf.out_fp4, buf.scales_fp4)
    calls["combine"] = lambda: B.moe_combine(prob, d_x, d_gates, buf.pair_slot, d_y)
    names = list(calls)
    trio = ["layout", "permute_bf16", "combine"]

    def timed(seq, per_kernel):
        for _ in range(3):
            flush_l2()
            for nm in seq:
                calls[nm]()
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(len(seq) + 1)]
              for _ in range(n_steps)]
        torch.cuda.synchronize(dev)
        for i in range(n_steps):
            flush_l2()
            ev[i][0].record(stream)
            for j, nm in enumerate(seq):
                calls[nm]()
                if per_kernel or j == len(seq) - 1:
                    ev[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
        if per_kernel:
            return [1e3 * sum(e[j].elapsed_time(e[j + 1]) for e in ev) / n_steps
                    for j in range(len(seq))]
        return 1e3 * sum(e[0].elapsed_time(e[-1]) for e in ev) / n_steps

    step_us = timed(names, False)
    trio_us = timed(trio, False)
    per = dict(zip(names, timed(names, True)))

    # launch-bound sizes (decode): the same step captured once into a CUDA
    # graph and replayed, as a serving loop would run it
    graph_us = None
    if w.P <= 4096:
        side = torch.cuda.Stream(device=dev)
        side.wait_stream(torch.cuda.current_stream(dev))
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=side):
            for nm in names:
                calls[nm]()
        for _ in range(3):
            flush_l2()
            graph.replay()
        ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
              for _ in range(n_steps)]
        torch.cuda.synchronize(dev)
        for a, b in ev:
            flush_l2()
            a.record(stream)
            graph.replay()
            b.record(stream)
        torch.cuda.synchronize(dev)
        graph_us = 1e3 * sum(a.elapsed_time(b) for a, b in ev) / n_steps
        del graph
        # one trivial kernel (a 4-byte fill) between two events after the same
        # flush: the launch and event cost that each of the phases above
        # carries when it is timed alone between events
        one = torch.zeros(1, dtype=torch.int32, device=dev)
        torch.cuda.synchronize(dev)
        for a, b in ev:
            flush_l2()
            a.record(stream)
            one.fill_(1)
            b.record(stream)
        torch.cuda.synchronize(dev)
        floor_us = 1e3 * sum(a.elapsed_time(b) for a, b in ev) / n_steps
    status = int(buf.status.cpu().numpy().view(np.uint32)[0])
    total_rows = int(buf.expert_counts.sum().item())
    nbytes = algorithmic_bytes(w, total_rows)
    step_bytes = sum(nbytes[nm] for nm in names)
    tiles = (w.P + 4095) // 4096
    out = {
        "workload": workload_config(w)["workload"],
        "layout_mode": (f"capacity [E, {w.expert_capacity}, H], drops in (token, k) order"
                        if w.expert_capacity > 0 else "packed, dropless"),
        "routed_rows": total_rows, "steps": n_steps,
        "step": " + ".join(names),
        "step_us": round(step_us, 2), "step_tokens_per_s": w.N / (step_us * 1e-6),
        "step_gbs": round(step_bytes / (step_us * 1e-6) / 1e9, 1),
        "step_frac_of_peak": round(step_bytes / (step_us * 1e-6) / 1e9 / peak, 3),
        "dispatch_bf16_plus_combine_us": round(trio_us, 2),
        "dispatch_bf16_plus_combine_tokens_per_s": w.N / (trio_us * 1e-6),
        "phases_us": {nm: round(v, 2) for nm, v in per.items()},
        "phases_gbs": {nm: round(nbytes[nm] / (per[nm] * 1e-6) / 1e9, 1) for nm in names},
        "phases_frac_of_peak": {nm: round(nbytes[nm] / (per[nm] * 1e-6) / 1e9 / peak, 3)
                                for nm in names},
        "algorithmic_bytes": {nm: nbytes[nm] for nm in names},
        "launches_per_step": layout_launches(w.P) + len(names) - 1,
        "layout_status": status,
    }
    if graph_us is not None:
        out["graph_step_us"] = round(graph_us, 2)
        out["graph_step_tokens_per_s"] = w.N / (graph_us * 1e-6)
        out["trivial_kernel_between_events_us"] = round(floor_us, 2)
    del buf, d_ids, d_hidden, d_gates, d_x, d_gs, d_y
    return out


def layout_launches(P: int) -> int:
    """Kernel launches of one moe_dispatch_layout call: one up to 128 tiles
    of 4096 pairs (the one-CTA, cluster or cooperative look-back kernel),
    else a scan and an emit launch."""
    return 1 if (P + 4095) // 4096 <= 128 else 2


def workload_config(w) -> dict:
    return {"workload": f"{w.name}: N={w.N} H={w.H} E={w.E} top_k={w.k} S={w.S} "
                        f"recv_capacity={w.recv_capacity}",
            "N": w.N, "H": w.H, "E": w.E, "top_k": w.k, "segments": w.S,
            "recv_capacity": w.recv_capacity,
            "step": "layout + permute(bf16) + permute(fp8 1x128) + permute(nvfp4) + combine",
            "l2": "flushed before every step (write of a 2x-L2 buffer, then a read of another "
                  "2x-L2 buffer to retire the dirty lines), outside the timed events",
            "parallelism": "replicas (independent token batches per GPU)"}


# ------------------------------------------------------------------ ours
def run_ours(args, rank: int, world: int, local: int) -> int:
    import torch
    import torch.distributed as dist

    from combine_topk_ids_scan_b200 import binding as B
    from combine_topk_ids_scan_b200.inputs import make_workload

    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        import datetime
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)

    def barrier():
        if world > 1:
            dist.barrier()

    B.load()
    w = make_workload(WORKLOAD, seed=seed_for_rank(rank))
    prob = B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity)
    buf = B.Buffers(prob, device=dev)
    stream = torch.cuda.current_stream(dev)

    # host inputs (pinned) and their device copies
    h_ids = torch.from_numpy(w.ids).pin_memory()
    h_hidden = torch.from_numpy(w.hidden.view(np.int16)).pin_memory()
    h_gates = torch.from_numpy(w.gates).pin_memory()
    h_x = torch.from_numpy(w.expert_out.view(np.int16))
    h_gs = torch.tensor([w.global_scale], dtype=torch.float32).pin_memory()
    d_ids = h_ids.to(dev)
    d_hidden = h_hidden.to(dev).view(torch.bfloat16)
    d_gates = h_gates.to(dev)
    d_x = h_x.to(dev).view(torch.bfloat16)
    d_gs = h_gs.to(dev)
    d_y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    h_y = torch.empty((w.N, w.H), dtype=torch.int16).pin_memory()
    h_status = torch.empty(1 + w.E, dtype=torch.int32).pin_memory()
    l2 = torch.cuda.get_device_properties(dev).L2_cache_size
    flush_w = torch.empty(max(2 * l2, 256 << 20), dtype=torch.uint8,
                          device=dev)
    flush_r = torch.zeros(max(2 * l2, 256 << 20) // 4, dtype=torch.int32, device=dev)

    def flush_l2():
        # write a buffer twice the L2 size, then read another one so the
        # dirty lines are written back here, outside the timed events
        flush_w.zero_()
        flush_r.max()

    def step(ev=None, phase_events=False):
        """One step; ev[0] / ev[5] bracket it, ev[1..4] (only with
        phase_events) separate its kernels.  An event between two kernels
        ends the programmatic overlap of the second with the first, so the
        timed steps record only the bracketing pair."""
        def mark(i):
            if ev is not None and (phase_events or i in (0, 5)):
                ev[i].record(stream)
        mark(0)
        B.layout(prob, d_ids, buf)
        mark(1)
        B.moe_permute(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out)
        mark(2)
        B.moe_permute_quant_fp8(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out_fp8,
                                buf.scales_fp8)
        mark(3)
        B.moe_permute_quant_nvfp4(prob, d_hidden, buf.row_src, buf.pair_slot, d_gs,
                                  buf.out_fp4, buf.scales_fp4)
        mark(4)
        B.moe_combine(prob, d_x, d_gates, buf.pair_slot, d_y)
        mark(5)

    # the layout's launches, then three permutes and the combine
    launches_per_step = layout_launches(w.P) + 4
    for _ in range(args.warmup):
        flush_l2()
        step()
    torch.cuda.synchronize(dev)
    st = int(buf.status.cpu().numpy().view(np.uint32)[0])
    total_rows = int(buf.expert_counts.sum().item())

    # ---- device-resident timed region
    uuid = None
    try:
        uuid = str(torch.cuda.get_device_properties(dev).uuid)
    except Exception:
        pass
    sampler = ClockSampler(uuid) if rank == 0 else None
    if sampler:
        sampler.start()
        time.sleep(0.3)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(args.steps)]
    barrier()
    torch.cuda.synchronize(dev)
    for i in range(args.steps):
        flush_l2()
        step(evs[i])
    torch.cuda.synchronize(dev)
    barrier()
    clocks = sampler.stop() if sampler else None
    step_ms = [e[0].elapsed_time(e[5]) for e in evs]
    ms = sum(step_ms) / len(step_ms)
    ms_median, ms_min = statistics.median(step_ms), min(step_ms)

    # ---- per-kernel breakdown: further steps with an event between kernels
    phases = ["layout", "permute_bf16", "permute_fp8", "permute_nvfp4", "combine"]
    n_phase = max(10, min(args.steps, 300))
    pevs = [[torch.cuda.Event(enable_timing=True) for _ in range(6)] for _ in range(n_phase)]
    torch.cuda.synchronize(dev)
    for i in range(n_phase):
        flush_l2()
        step(pevs[i], phase_events=True)
    torch.cuda.synchronize(dev)
    per = {p: [] for p in phases}
    for e in pevs:
        for i, p in enumerate(phases):
            per[p].append(e[i].elapsed_time(e[i + 1]))
    phase_ms = {p: sum(v) / len(v) for p, v in per.items()}
    phase_step_ms = sum(e[0].elapsed_time(e[5]) for e in pevs) / n_phase

    # ---- each kernel alone: the L2 flushed before every kernel (the dirty
    # lines the previous kernel left are written back inside the flush, not
    # inside the next kernel's events), as an ncu capture runs it
    calls = [lambda: B.layout(prob, d_ids, buf),
             lambda: B.moe_permute(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out),
             lambda: B.moe_permute_quant_fp8(prob, d_hidden, buf.row_src, buf.pair_slot,
                                             buf.out_fp8, buf.scales_fp8),
             lambda: B.moe_permute_quant_nvfp4(prob, d_hidden, buf.row_src, buf.pair_slot, d_gs,
                                               buf.out_fp4, buf.scales_fp4),
             lambda: B.moe_combine(prob, d_x, d_gates, buf.pair_slot, d_y)]
    n_alone = max(10, min(args.steps, 100))
    aev = [[(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
            for _ in calls] for _ in range(n_alone)]
    torch.cuda.synchronize(dev)
    for i in range(n_alone):
        for j, c in enumerate(calls):
            flush_l2()
            aev[i][j][0].record(stream)
            c()
            aev[i][j][1].record(stream)
    torch.cuda.synchronize(dev)
    alone_ms = {p: sum(aev[i][j][0].elapsed_time(aev[i][j][1]) for i in range(n_alone)) / n_alone
                for j, p in enumerate(phases)}

    def time_phases(calls, n_steps):
        """Average device time (us) of each call in `calls`, run in order as
        one step; L2 flushed before every step, 3 untimed warm-up steps."""
        for _ in range(3):
            flush_l2()
            for c in calls:
                c()
        evp = [[torch.cuda.Event(enable_timing=True) for _ in range(len(calls) + 1)]
               for _ in range(n_steps)]
        torch.cuda.synchronize(dev)
        for i in range(n_steps):
            flush_l2()
            evp[i][0].record(stream)
            for j, c in enumerate(calls):
                c()
                evp[i][j + 1].record(stream)
        torch.cuda.synchronize(dev)
        return [1e3 * sum(e[j].elapsed_time(e[j + 1]) for e in evp) / n_steps
                for j in range(len(calls))]

    # ---- grouped-GEMM-ready dispatch (NEXT row f1): experts padded to 128
    # rows, NVFP4 scales in the 128x4 atom layout; recv_capacity covers the
    # worst case N*k + E*127 and every one of its rows is written
    f1 = None
    if args.next_rows:
        pad = 128
        prob_p = B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                           num_segments=w.S, recv_capacity=w.N * w.k + w.E * (pad - 1),
                           flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES, expert_pad_multiple=pad)
        buf_p = B.Buffers(prob_p, device=dev)
        f1_steps = max(10, args.steps // 10)
        lay_us, nv_us = time_phases(
            [lambda: B.layout(prob_p, d_ids, buf_p),
             lambda: B.moe_permute_quant_nvfp4(prob_p, d_hidden, buf_p.row_src, buf_p.pair_slot,
                                               d_gs, buf_p.out_fp4, buf_p.scales_fp4)],
            f1_steps)
        rows_p = buf_p.rows
        nv_bytes = (2 * w.N * w.H + 4 * w.P + 4 * rows_p + rows_p * w.H // 2
                    + B.nvfp4_swizzled_scale_bytes(rows_p, w.H) + 4)
        padded_total = int(buf_p.expert_offsets[-1].item())
        f1 = {"expert_pad_multiple": pad, "recv_capacity": rows_p,
              "padded_rows_routed": padded_total, "steps": f1_steps,
              "layout_us": round(lay_us, 2), "permute_nvfp4_swizzled_us": round(nv_us, 2),
              "permute_nvfp4_swizzled_gbs": round(nv_bytes / (nv_us * 1e-6) / 1e9, 1),
              "tokens_per_s": w.N / ((lay_us + nv_us) * 1e-6)}
        del buf_p

    # ---- expert-parallel send fused into the permute (NEXT row f2): segment
    # s of the dispatch goes straight into "rank" s's receive buffer; on one
    # GPU the S receive buffers are local stand-ins for the peers' buffers
    f2 = None
    if args.next_rows:
        meta_h = buf.meta.cpu().numpy().view(np.uint32)
        seg_rows = [int(v) // w.H for v in meta_h[0]]
        recv = [torch.empty((max(r, 1), w.H), dtype=torch.bfloat16, device=dev)
                for r in seg_rows]
        peer = torch.tensor([t.data_ptr() for t in recv], dtype=torch.int64, device=dev)
        put = torch.zeros(w.S, dtype=torch.int64, device=dev)
        f2_steps = max(10, args.steps // 10)
        # the quantised forms: codes and scales per receiver
        r8 = [(torch.empty((max(r, 1), w.H), dtype=torch.uint8, device=dev),
               torch.empty((max(r, 1), w.H // 128), dtype=torch.float32, device=dev))
              for r in seg_rows]
        r4 = [(torch.empty((max(r, 1), w.H // 2), dtype=torch.uint8, device=dev),
               torch.empty((max(r, 1), w.H // 16), dtype=torch.uint8, device=dev))
              for r in seg_rows]

        def ptrs(bufs, i):
            return torch.tensor([b[i].data_ptr() for b in bufs], dtype=torch.int64, device=dev)

        c8, s8, c4, s4 = ptrs(r8, 0), ptrs(r8, 1), ptrs(r4, 0), ptrs(r4, 1)
        pp_us, p8_us, p4_us = time_phases(
            [lambda: B.moe_permute_to_peers(prob, d_hidden, buf.row_src, buf.pair_slot,
                                            buf.meta, peer, put),
             lambda: B.moe_permute_quant_fp8_to_peers(prob, d_hidden, buf.row_src,
                                                      buf.pair_slot, buf.meta, c8, s8, put),
             lambda: B.moe_permute_quant_nvfp4_to_peers(prob, d_hidden, buf.row_src,
                                                        buf.pair_slot, buf.meta, d_gs, c4, s4,
                                                        put)], f2_steps)
        # the return: every rank's combine reads the expert outputs straight
        # from the owners' buffers (here the bf16 receive buffers the send
        # just filled: identity experts)
        (cp_us,) = time_phases([lambda: B.moe_combine_from_peers(
            prob, peer, put, buf.meta, d_gates, buf.pair_slot, d_y)], f2_steps)
        cp_bytes = (2 * int(buf.expert_counts.sum().item()) * w.H + 8 * w.P
                    + 2 * w.N * w.H)       # the combine's algorithmic bytes
        maps = 2 * w.N * w.H + 4 * w.P + 4 * buf.rows + 16 * w.S
        routed = sum(seg_rows)
        pp_bytes = maps + 2 * routed * w.H
        p8_bytes = maps + routed * (w.H + 4 * (w.H // 128))
        p4_bytes = maps + routed * (w.H // 2 + w.H // 16) + 4
        f2 = {"steps": f2_steps, "segments": w.S,
              "permute_to_peers_us": round(pp_us, 2),
              "permute_to_peers_gbs": round(pp_bytes / (pp_us * 1e-6) / 1e9, 1),
              "permute_fp8_to_peers_us": round(p8_us, 2),
              "permute_fp8_to_peers_gbs": round(p8_bytes / (p8_us * 1e-6) / 1e9, 1),
              "permute_nvfp4_to_peers_us": round(p4_us, 2),
              "permute_nvfp4_to_peers_gbs": round(p4_bytes / (p4_us * 1e-6) / 1e9, 1),
              "combine_from_peers_us": round(cp_us, 2),
              "combine_from_peers_gbs": round(cp_bytes / (cp_us * 1e-6) / 1e9, 1),
              "receivers": "S local buffers standing in for the peers' receive buffers "
                           "(one GPU); across GPUs the same stores go over NVLink"}
        del recv, peer, put, r8, r4, c8, s8, c4, s4

    # ---- backward (NEXT row f4): dispatch backward (gather-sum of the rows'
    # gradients) and combine backward (scaled scatter + gate gradients)
    f4 = None
    if args.next_rows:
        d_grows = d_x                      # a [C, H] bf16 gradient of the dispatch output
        d_gtok = d_hidden                  # an [N, H] bf16 gradient of the combine output
        d_gh = torch.empty_like(d_hidden)
        d_gx = torch.empty_like(d_x)
        d_gw = torch.empty_like(d_gates)
        f4_steps = max(10, args.steps // 10)
        pb_us, cb_us, pm_us = time_phases(
            [lambda: B.moe_permute_backward(prob, d_grows, buf.pair_slot, d_gh),
             lambda: B.moe_combine_backward(prob, d_gtok, d_x, d_gates, buf.pair_slot,
                                            buf.row_src, d_gx, d_gw),
             lambda: B.moe_permute_premultiplied(prob, d_hidden, buf.row_src, buf.pair_slot,
                                                 d_gates, d_gx)],
            f4_steps)
        rows = buf.rows
        pb_bytes = 2 * total_rows * w.H + 4 * w.P + 2 * w.N * w.H
        cb_bytes = (2 * w.N * w.H + 2 * 2 * total_rows * w.H + 2 * (rows - total_rows) * w.H
                    + 4 * w.P * 3 + 4 * rows)
        pm_bytes = 2 * w.N * w.H + 4 * w.P + 4 * rows + 4 * w.P + 2 * rows * w.H
        f4 = {"steps": f4_steps,
              "permute_premultiplied_us": round(pm_us, 2),
              "permute_premultiplied_gbs": round(pm_bytes / (pm_us * 1e-6) / 1e9, 1),
              "permute_backward_us": round(pb_us, 2),
              "permute_backward_gbs": round(pb_bytes / (pb_us * 1e-6) / 1e9, 1),
              "combine_backward_us": round(cb_us, 2),
              "combine_backward_gbs": round(cb_bytes / (cb_us * 1e-6) / 1e9, 1),
              "tokens_per_s": w.N / ((pb_us + cb_us) * 1e-6)}
        del d_gh, d_gx, d_gw

    # ---- MX token format and fused SwiGLU + requantisation (NEXT row f3):
    # the MXFP4 dispatch of the same tokens, and the synthetic expert outputs
    # [C, H] read as gate|up rows of intermediate size I = H / 2
    f3 = None
    if args.next_rows:
        n3 = max(10, args.steps // 20)
        (mx_us,) = time_phases([lambda: B.moe_permute_quant_mxfp4(
            prob, d_hidden, buf.row_src, buf.pair_slot, buf.out_mx4, buf.scales_mx4)], n3)
        mx_bytes = (2 * w.N * w.H + 4 * w.P + 4 * buf.rows + buf.rows * w.H // 2
                    + buf.rows * w.H // 32)
        I = w.H // 2
        f3 = {"permute_mxfp4_us": round(mx_us, 2),
              "permute_mxfp4_gbs": round(mx_bytes / (mx_us * 1e-6) / 1e9, 1),
              "swiglu": {"intermediate": I, "gate_up": "split", "rows": buf.rows}}
        for fmt, name in ((B.MOE_QUANT_MXFP8, "mxfp8"), (B.MOE_QUANT_NVFP4, "nvfp4"),
                          (B.MOE_QUANT_MXFP4, "mxfp4"), (B.MOE_QUANT_MXFP6_E2M3, "mxfp6_e2m3"),
                          (B.MOE_QUANT_BF16, "bf16")):
            codes, scales = B.swiglu_buffers(buf.rows, I, fmt, device=dev)
            (us,) = time_phases([lambda: B.moe_swiglu_quant(
                prob, I, fmt, B.MOE_GATE_UP_SPLIT, d_x, buf.row_src, d_gs, codes, scales)], n3)
            nbytes = (2 * 2 * I * total_rows + 4 * buf.rows + codes.numel()
                      + (scales.numel() if fmt != B.MOE_QUANT_BF16 else 0))
            f3["swiglu"][name + "_us"] = round(us, 2)
            f3["swiglu"][name + "_gbs"] = round(nbytes / (us * 1e-6) / 1e9, 1)
            del codes, scales

    # ---- every workload of the benchmark set, each timed alone beside the
    # oracle on a bounded sample of it (one GPU only: a per-rank sweep would
    # only repeat it)
    configs = None
    if args.configs and world == 1:
        peak_c, _ = _peaks()
        configs = {}
        n_cfg = max(20, min(args.steps, 100))
        for name in CONFIG_SET:
            wc = w if name == WORKLOAD else make_workload(name)
            r = measure_workload(B, torch, wc, dev, stream, flush_l2, n_cfg, peak_c)
            if not args.no_cpu_baseline:
                n_cpu = min(CPU_SAMPLE_TOKENS[name], wc.N)
                tps, dt = oracle_tokens_per_s(wc, n_cpu)
                r["cpu_baseline"] = {"value": tps, "unit": "tokens/s", "cores": 1,
                                     "kind": "oracle",
                                     "sample": f"first {n_cpu} tokens, own layout; "
                                               f"{dt:.2f} s single-threaded"}
                r["gpu_vs_cpu_step"] = r["step_tokens_per_s"] / tps
            configs[name] = r
            if wc is not w:
                del wc

    # ---- end to end through the public API from pinned host memory
    # Every step: H2D of the step's inputs (ids, hidden rows, gates, global
    # scale), the whole path with identity experts (the combine reads the bf16
    # dispatch output), D2H of the combined rows, the status word and the
    # counts.  Three input/output sets and three streams let the next steps'
    # H2D and the previous steps' D2H overlap step i, as a serving loop would.
    e2e_steps = max(4, min(args.steps, 40))
    NSETS = 3
    h_y2 = [h_y] + [torch.empty_like(h_y).pin_memory() for _ in range(NSETS - 1)]
    h_st2 = [h_status] + [torch.empty_like(h_status).pin_memory() for _ in range(NSETS - 1)]
    sets = [dict(ids=torch.empty_like(d_ids), hidden=torch.empty_like(d_hidden),
                 gates=torch.empty_like(d_gates), gs=torch.empty_like(d_gs),
                 y=torch.empty_like(d_y), st=torch.empty(1 + w.E, dtype=torch.int32, device=dev))
            for _ in range(NSETS)]
    s_in, s_comp, s_out = (torch.cuda.Stream(dev) for _ in range(3))
    ev_in = [torch.cuda.Event() for _ in range(NSETS)]
    ev_comp = [torch.cuda.Event() for _ in range(NSETS)]
    ev_out = [torch.cuda.Event() for _ in range(NSETS)]
    h2d = h_ids.numel() * 4 + h_hidden.numel() * 2 + h_gates.numel() * 4 + h_gs.numel() * 4
    d2h = h_y.numel() * 2 + h_status.numel() * 4

    def e2e_step(i):
        b = i % NSETS
        S = sets[b]
        with torch.cuda.stream(s_in):
            if i >= NSETS:
                s_in.wait_event(ev_comp[b])      # step i-NSETS is done with set b's inputs
            S["ids"].copy_(h_ids, non_blocking=True)
            S["hidden"].view(torch.int16).copy_(h_hidden, non_blocking=True)
            S["gates"].copy_(h_gates, non_blocking=True)
            S["gs"].copy_(h_gs, non_blocking=True)
            ev_in[b].record(s_in)
        with torch.cuda.stream(s_comp):
            s_comp.wait_event(ev_in[b])
            if i >= NSETS:
                s_comp.wait_event(ev_out[b])     # set b's result has been read out
            B.layout(prob, S["ids"], buf)
            B.moe_permute(prob, S["hidden"], buf.row_src, buf.pair_slot, buf.out)
            B.moe_permute_quant_fp8(prob, S["hidden"], buf.row_src, buf.pair_slot, buf.out_fp8,
                                    buf.scales_fp8)
            B.moe_permute_quant_nvfp4(prob, S["hidden"], buf.row_src, buf.pair_slot, S["gs"],
                                      buf.out_fp4, buf.scales_fp4)
            B.moe_combine(prob, buf.out, S["gates"], buf.pair_slot, S["y"])
            S["st"][:1].copy_(buf.status)
            S["st"][1:].copy_(buf.expert_counts)
            ev_comp[b].record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(ev_comp[b])
            h_y2[b].copy_(S["y"].view(torch.int16), non_blocking=True)
            h_st2[b].copy_(S["st"], non_blocking=True)
            ev_out[b].record(s_out)

    for i in range(2 * NSETS):                   # warm the streams and sets
        e2e_step(i)
    torch.cuda.synchronize(dev)
    e_start = torch.cuda.Event(enable_timing=True)
    e_end = torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e_start.record(s_in)
    for i in range(e2e_steps):
        e2e_step(i)
    s_out.wait_stream(s_in)
    s_out.wait_stream(s_comp)
    e_end.record(s_out)
    torch.cuda.synchronize(dev)
    barrier()
    e2e_ms = e_start.elapsed_time(e_end) / e2e_steps

    # ---- max over ranks
    t = max_over_ranks([ms, e2e_ms] + [phase_ms[p] for p in phases], dev, world)
    ms, e2e_ms = t[0], t[1]
    phase_ms = {p: t[2 + i] for i, p in enumerate(phases)}

    if rank == 0:
        nbytes = algorithmic_bytes(w, total_rows)
        step_bytes = sum(nbytes.values())
        peak, peak_kind = _peaks()
        dom = max(("permute_bf16", "permute_fp8", "permute_nvfp4", "combine"),
                  key=lambda p: phase_ms[p])
        achieved = nbytes[dom] / (phase_ms[dom] * 1e-3) / 1e9
        tr = NCU_TRAFFIC.get(dom)
        traffic = tr["bytes_per_launch"] if tr and tr.get("src_sha") == _kernel_src_sha(dom) \
            else None
        value = world * w.N / (ms * 1e-3)
        line = {
            "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "ms_per_step_median": ms_median, "ms_per_step_min": ms_min,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp32", "data": "synthetic", "config": workload_config(w),
            "hbm_gbs": step_bytes / (ms * 1e-3) / 1e9,
            "hbm_frac_of_peak": step_bytes / (ms * 1e-3) / 1e9 / peak,
            "hbm_frac_of_nominal": step_bytes / (ms * 1e-3) / 1e9 / NOMINAL_HBM_GBS,
            "phases_us": {p: round(1e3 * v, 2) for p, v in phase_ms.items()},
            "phases_timing": (f"{n_phase} further steps with an event between kernels (an event "
                              f"ends the programmatic overlap of consecutive kernels); their "
                              f"mean step {phase_step_ms:.4f} ms"),
            "phases_gbs": {p: round(nbytes[p] / (phase_ms[p] * 1e-3) / 1e9, 1)
                           for p in phases},
            "phases_alone_us": {p: round(1e3 * v, 2) for p, v in alone_ms.items()},
            "phases_alone_gbs": {p: round(nbytes[p] / (alone_ms[p] * 1e-3) / 1e9, 1)
                                 for p in phases},
            "phases_alone_timing": (f"{n_alone} more passes, each kernel alone: the L2 flushed "
                                    "before every kernel, one event pair around it (context; the "
                                    "roofline uses the in-step phases above)"),
            "dispatch_bf16_plus_combine_tokens_per_s":
                world * w.N / ((phase_ms["layout"] + phase_ms["permute_bf16"]
                                + phase_ms["combine"]) * 1e-3),
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "peak_source": f"{peak_kind} hbm_gbs", "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes": nbytes[dom]},
            "e2e": {"value": world * w.N / (e2e_ms * 1e-3), "unit": "tokens/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "ms_per_step": e2e_ms,
                    "path": "pinned host -> H2D -> layout, 3 permutes, combine (identity "
                            "experts: combine reads the bf16 dispatch output) -> D2H of the "
                            "combined rows, status and counts; copies of neighbouring steps "
                            "overlap on separate streams"},
            "gpu_launches": launches_per_step * args.steps,
            "next_rows": ({"f1_grouped_gemm_ready_nvfp4": f1,
                           "f2_permute_to_peers": f2, "f3_mx_and_swiglu_requant": f3,
                           "f4_backward": f4} if f1 or f2 or f3 or f4 else None),
            "configs": configs,
            "clocks": clocks, "layout_status": st,
        }
        if world == 1 and not args.no_cpu_baseline:
            n_cpu = args.cpu_tokens
            tps, dt = oracle_tokens_per_s(w, n_cpu)
            box = os.cpu_count() or 1
            tps_all, dt_all = oracle_tokens_per_s(w, n_cpu, threads=box)
            line["cpu_baseline"] = {
                "value": tps, "unit": "tokens/s", "cores": 1, "kind": "oracle",
                "sample": f"first {n_cpu} tokens of the batch, own layout with "
                          f"recv_capacity = {n_cpu}*k; {dt:.1f} s single-threaded",
                "box_cores": box,
                "all_cores": {"value": tps_all, "unit": "tokens/s", "threads": box,
                              "seconds": round(dt_all, 2),
                              "how": "the same oracle calls, the permutes' rows and the "
                                     "combine's tokens split over a thread pool"}}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main() -> int:
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--cpu-tokens", type=int, default=2048)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-next-rows", dest="next_rows", action="store_false",
                    help="skip the extra measurement of the grouped-GEMM-ready dispatch")
    ap.add_argument("--no-configs", dest="configs", action="store_false",
                    help="skip the sweep over every workload of the benchmark set")
    args = ap.parse_args()
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank, world, local = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)
    return run_ours(args, rank, world, local)


if __name__ == "__main__":
    sys.exit(main())
