"""Per-CTA trace records of the build with -DMOE_TRACE (libmoedc_trace.so).

The library's kernels append one 32-byte record per CTA (moe_trace_record in
include/moe_dc.h: start and end on the GPU's nanosecond timer, launch id,
block index, SM, kernel id and variant) to a buffer attached with
moe_trace_attach.  This module decodes the records on the host and groups
them into launches; Tracer attaches a buffer around a block of calls:

    from combine_topk_ids_scan_b200 import binding as B, trace
    with trace.Tracer(capacity=1 << 16) as tr:     # MOE_LIB_PATH = the trace build
        B.layout(prob, ids, buf)
        B.moe_permute(prob, hidden, buf.row_src, buf.pair_slot, buf.out)
    for launch in tr.launches():
        print(launch.kernel, launch.ctas, launch.duration_us)

`python -m combine_topk_ids_scan_b200.trace [--workload NAME] [--steps K]`
builds and loads the trace build and prints the per-kernel timeline of one
benchmark step (layout, bf16 / FP8 / NVFP4 permutes, combine) on a seeded
workload, the L2 flushed before every step.
"""
from __future__ import annotations

import argparse
import statistics
from dataclasses import dataclass

import numpy as np

RECORD_DTYPE = np.dtype([("start_ns", "<u8"), ("end_ns", "<u8"), ("grid", "<u8"),
                         ("block", "<u4"), ("smid", "<u2"), ("kernel", "u1"),
                         ("variant", "u1")])
assert RECORD_DTYPE.itemsize == 32

# moe_trace_kernel
KERNELS = {
    1: "layout_single", 2: "layout_cluster", 3: "layout_lookback", 4: "layout_scan",
    5: "layout_emit", 6: "permute_bf16", 7: "permute_fp8", 8: "permute_nvfp4",
    9: "permute_mxfp4", 10: "scales_to_atoms", 11: "permute_premultiplied",
    12: "permute_to_peers", 13: "combine", 14: "permute_backward", 15: "combine_backward",
    16: "swiglu_split", 17: "swiglu_quant", 18: "permute_fp8_to_peers",
    19: "permute_nvfp4_to_peers", 20: "combine_from_peers",
}
LAYOUT_KERNELS = frozenset(range(1, 6))


@dataclass(frozen=True)
class Launch:
    """The CTAs of one kernel launch: one %gridid, and the instance-th launch
    with that id (replays of a captured CUDA graph reuse their kernel node's
    id)."""
    kernel: str
    kernel_id: int
    variant: int
    grid: int
    instance: int
    ctas: int
    sms: int          # distinct SMs its CTAs ran on
    start_ns: int     # earliest CTA start
    end_ns: int       # latest CTA end

    @property
    def duration_us(self) -> float:
        return (self.end_ns - self.start_ns) / 1e3


def decode(raw: np.ndarray, count: int) -> np.ndarray:
    """The records a traced run wrote: `raw` is the record buffer's bytes
    (uint8, capacity * 32), `count` the device counter's final value.
    Records past the capacity were dropped by the kernels."""
    raw = np.ascontiguousarray(raw).view(np.uint8).reshape(-1)
    capacity = raw.size // RECORD_DTYPE.itemsize
    recs = raw[:capacity * RECORD_DTYPE.itemsize].view(RECORD_DTYPE)
    return recs[:min(int(count), capacity)].copy()


def dropped(count: int, capacity: int) -> int:
    """Records the kernels could not write (count ran past the capacity)."""
    return max(0, int(count) - int(capacity))


def instances(records: np.ndarray) -> np.ndarray:
    """Launch instance of each record: how many earlier records (in slot
    order, which is the order the CTAs started) have its %gridid and block.
    A grid id recurs when a captured CUDA graph is replayed; the n-th replay's
    CTAs all start after the (n-1)-th replay's have finished."""
    n = records.size
    slot = np.arange(n)
    order = np.lexsort((slot, records["block"], records["grid"]))
    g, b = records["grid"][order], records["block"][order]
    new = np.ones(n, bool)
    new[1:] = (g[1:] != g[:-1]) | (b[1:] != b[:-1])
    first = np.maximum.accumulate(np.where(new, slot, 0))
    inst = np.empty(n, np.int64)
    inst[order] = slot - first
    return inst


def records_of(records: np.ndarray, launch: Launch) -> np.ndarray:
    """The records of one launch."""
    return records[(records["grid"] == launch.grid) & (instances(records) == launch.instance)]


def launches(records: np.ndarray) -> list[Launch]:
    """Group records by launch, in the order the launches started."""
    inst = instances(records)
    out = []
    for g in np.unique(records["grid"]):
        for i in np.unique(inst[records["grid"] == g]):
            r = records[(records["grid"] == g) & (inst == i)]
            kid = int(r["kernel"][0])
            if np.any(r["kernel"] != kid) or np.any(r["variant"] != r["variant"][0]):
                raise ValueError(f"launch {int(g)}.{int(i)} mixes kernel ids or variants")
            out.append(Launch(kernel=KERNELS.get(kid, f"kernel{kid}"), kernel_id=kid,
                              variant=int(r["variant"][0]), grid=int(g), instance=int(i),
                              ctas=int(r.size), sms=int(np.unique(r["smid"]).size),
                              start_ns=int(r["start_ns"].min()),
                              end_ns=int(r["end_ns"].max())))
    out.sort(key=lambda launch: (launch.start_ns, launch.grid, launch.instance))
    return out


class Tracer:
    """Attach a record buffer of `capacity` records on entry (on the current
    stream), detach and read the records back on exit."""

    def __init__(self, capacity: int = 1 << 16, stream=None):
        self.capacity = int(capacity)
        self.stream = stream
        self.count = 0
        self._records = None

    def __enter__(self) -> "Tracer":
        import torch

        from combine_topk_ids_scan_b200 import binding as B
        self._raw = torch.zeros(self.capacity * RECORD_DTYPE.itemsize, dtype=torch.uint8,
                                device="cuda")
        self._count = torch.zeros(1, dtype=torch.int32, device="cuda")
        B.moe_trace_attach(self._raw, self._count, self.stream)
        return self

    def __exit__(self, *exc) -> None:
        import torch

        from combine_topk_ids_scan_b200 import binding as B
        B.moe_trace_attach(None, None, self.stream)
        torch.cuda.synchronize()
        self.count = int(self._count.cpu().numpy().view(np.uint32)[0])
        self._records = decode(self._raw.cpu().numpy(), self.count)

    @property
    def dropped(self) -> int:
        return dropped(self.count, self.capacity)

    def records(self) -> np.ndarray:
        return self._records

    def launches(self) -> list[Launch]:
        return launches(self._records)


def _step_calls(B, torch, w):
    """The benchmark step's calls on device copies of workload w."""
    dev = torch.device("cuda", torch.cuda.current_device())

    def bf16(a):
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).to(dev).view(
            torch.bfloat16)

    prob = B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity)
    buf = B.Buffers(prob, device=dev)
    ids = torch.from_numpy(w.ids).to(dev)
    hidden, x = bf16(w.hidden), bf16(w.expert_out)
    gates = torch.from_numpy(w.gates).to(dev)
    gs = torch.tensor([w.global_scale], dtype=torch.float32, device=dev)
    y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device=dev)
    calls = [lambda: B.layout(prob, ids, buf),
             lambda: B.moe_permute(prob, hidden, buf.row_src, buf.pair_slot, buf.out)]
    if w.H % 128 == 0:
        calls.append(lambda: B.moe_permute_quant_fp8(prob, hidden, buf.row_src, buf.pair_slot,
                                                     buf.out_fp8, buf.scales_fp8))
    if w.H % 32 == 0:
        calls.append(lambda: B.moe_permute_quant_nvfp4(prob, hidden, buf.row_src,
                                                       buf.pair_slot, gs, buf.out_fp4,
                                                       buf.scales_fp4))
    calls.append(lambda: B.moe_combine(prob, x, gates, buf.pair_slot, y))
    return calls, (buf, ids, hidden, x, gates, gs, y)


def main(argv=None) -> None:
    from combine_topk_ids_scan_b200.inputs import CONFIG_NAMES, make_workload
    ap = argparse.ArgumentParser(description=__doc__.split("\n")[0])
    ap.add_argument("--workload", default="fp8_metric", choices=CONFIG_NAMES)
    ap.add_argument("--steps", type=int, default=10)
    a = ap.parse_args(argv)

    import torch

    from combine_topk_ids_scan_b200 import binding as B
    from combine_topk_ids_scan_b200 import build
    B.load(build.build(trace=True))
    if "trace records" not in B.version():
        raise SystemExit(f"not the trace build: {B.version()}")
    w = make_workload(a.workload)
    calls, _keep = _step_calls(B, torch, w)
    l2 = torch.cuda.get_device_properties(0).L2_cache_size
    scratch = torch.empty(2 * l2, dtype=torch.uint8, device="cuda")
    for i in range(3):
        for c in calls:
            c()
    per: dict[tuple, list] = {}
    for i in range(a.steps):
        scratch.fill_(i & 0xFF)
        torch.cuda.synchronize()
        with Tracer(capacity=1 << 18) as tr:
            for c in calls:
                c()
        if tr.dropped:
            raise SystemExit(f"{tr.dropped} records dropped")
        prev_end = None
        for j, launch in enumerate(tr.launches()):
            # the kernel's own span: from the later of its first CTA's start
            # and the previous kernel's end (a dependent launch starts its
            # CTAs early, and they wait) to its last CTA's end
            own = launch.end_ns - (launch.start_ns if prev_end is None
                                   else max(launch.start_ns, prev_end))
            per.setdefault((j, launch.kernel, launch.variant), []).append(
                (own / 1e3, launch.duration_us, launch.ctas, launch.sms))
            prev_end = launch.end_ns
    print(f"workload {a.workload}: N={w.N} H={w.H} E={w.E} k={w.k}; {a.steps} steps, "
          f"L2 flushed before each; medians")
    print("| kernel | variant | CTAs | SMs | us after the previous kernel ended | "
          "us first CTA start to last CTA end |")
    print("|---|---|---|---|---|---|")
    for (j, name, var), v in sorted(per.items()):
        print(f"| {name} | {var} | {v[0][2]} | {v[0][3]} | "
              f"{statistics.median(x[0] for x in v):.1f} | "
              f"{statistics.median(x[1] for x in v):.1f} |")


if __name__ == "__main__":
    main()
