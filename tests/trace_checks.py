"""Consistency checks of the per-CTA trace records of one traced run
(combine_topk_ids_scan_b200.trace), shared by the trace-build tests."""
from __future__ import annotations

import numpy as np
import torch

from combine_topk_ids_scan_b200 import trace as T


def check_launches(tr: T.Tracer) -> list[T.Launch]:
    """Every CTA of every launch recorded exactly once with start <= end on a
    valid SM, and consecutive launches (one stream) in order: the later one's
    CTAs all start after every CTA of the earlier one started (a dependent
    launch is scheduled only once they all did), and all end after the
    earlier one's last CTA ended (each waits for the earlier grid)."""
    assert tr.dropped == 0, f"{tr.dropped} records dropped"
    recs = tr.records()
    sms = torch.cuda.get_device_properties(0).multi_processor_count
    assert np.all(recs["start_ns"] <= recs["end_ns"])
    assert np.all(recs["smid"] < sms)
    assert set(np.unique(recs["kernel"]).tolist()) <= set(T.KERNELS)
    ls = T.launches(recs)
    for launch in ls:
        blocks = np.sort(T.records_of(recs, launch)["block"])
        assert np.array_equal(blocks, np.arange(launch.ctas)), launch
    ordered = sorted(ls, key=lambda x: (x.start_ns, x.end_ns))
    for a, b in zip(ordered, ordered[1:]):
        ra = T.records_of(recs, a)
        rb = T.records_of(recs, b)
        assert int(rb["start_ns"].min()) >= int(ra["start_ns"].max()), (a, b)
        assert int(rb["end_ns"].min()) >= int(ra["end_ns"].max()), (a, b)
    return ordered
