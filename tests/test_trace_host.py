"""Host side of the trace records (combine_topk_ids_scan_b200/trace.py) on
hand-made record buffers, and the normal build's answer to moe_trace_attach
(no GPU needed)."""
import numpy as np
import pytest

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200 import build
from combine_topk_ids_scan_b200 import trace as T


def _rec(start, end, grid, block, smid, kernel, variant=0):
    r = np.zeros(1, T.RECORD_DTYPE)
    r[0] = (start, end, grid, block, smid, kernel, variant)
    return r


def test_record_layout_matches_the_c_struct():
    # moe_trace_record: three u64, u32 block, u16 smid, u8 kernel, u8 variant
    assert T.RECORD_DTYPE.itemsize == B.TRACE_RECORD_BYTES == 32
    assert [T.RECORD_DTYPE.fields[n][1] for n in T.RECORD_DTYPE.names] == \
        [0, 8, 16, 24, 28, 30, 31]


def test_decode_keeps_the_written_records_and_counts_the_dropped():
    recs = np.concatenate([_rec(10 + i, 20 + i, 7, i, i % 3, 6) for i in range(5)])
    raw = np.full(8 * 32, 0xA5, np.uint8)           # capacity 8, 5 written
    raw[:5 * 32] = recs.view(np.uint8)
    got = T.decode(raw, 5)
    assert got.size == 5 and np.array_equal(got, recs)
    # counter past the capacity: every slot holds a record, the rest dropped
    full = np.concatenate([recs, recs[:3]])
    got = T.decode(full.view(np.uint8), 11)
    assert got.size == 8
    assert T.dropped(11, 8) == 3 and T.dropped(5, 8) == 0


def test_launches_group_by_grid_in_start_order():
    recs = np.concatenate([
        _rec(500, 900, grid=42, block=1, smid=4, kernel=13, variant=8),
        _rec(100, 300, grid=41, block=0, smid=0, kernel=2, variant=4),
        _rec(480, 950, grid=42, block=0, smid=5, kernel=13, variant=8),
        _rec(110, 320, grid=41, block=1, smid=1, kernel=2, variant=4),
        _rec(120, 310, grid=41, block=2, smid=1, kernel=2, variant=4),
    ])
    ls = T.launches(recs)
    assert [launch.kernel for launch in ls] == ["layout_cluster", "combine"]
    a, b = ls
    assert (a.ctas, a.sms, a.start_ns, a.end_ns, a.variant) == (3, 2, 100, 320, 4)
    assert (b.ctas, b.sms, b.start_ns, b.end_ns, b.variant) == (2, 2, 480, 950, 8)
    assert b.duration_us == pytest.approx(0.47)


def test_a_recurring_grid_id_splits_into_launch_instances():
    # two replays of one captured graph node: the same grid id, blocks 0-1
    # twice, the second replay's CTAs in later slots
    recs = np.concatenate([_rec(10, 20, 5, 0, 0, 6), _rec(11, 21, 5, 1, 1, 6),
                           _rec(30, 40, 5, 1, 2, 6), _rec(31, 42, 5, 0, 3, 6)])
    assert T.instances(recs).tolist() == [0, 0, 1, 1]
    a, b = T.launches(recs)
    assert (a.instance, a.ctas, a.start_ns, a.end_ns) == (0, 2, 10, 21)
    assert (b.instance, b.ctas, b.start_ns, b.end_ns) == (1, 2, 30, 42)
    assert sorted(T.records_of(recs, b)["block"].tolist()) == [0, 1]


def test_a_launch_mixing_kernel_ids_is_rejected():
    recs = np.concatenate([_rec(1, 2, 9, 0, 0, 6), _rec(1, 2, 9, 1, 0, 7)])
    with pytest.raises(ValueError):
        T.launches(recs)


def test_kernel_names_cover_the_header_enum():
    import os
    import re
    hdr = open(os.path.join(os.path.dirname(build.PKG), "include", "moe_dc.h")).read()
    ids = {int(v) for v in re.findall(r"MOE_TRACE_\w+ = (\d+)", hdr)}
    assert ids == set(T.KERNELS)


def test_normal_build_answers_not_built_without_cuda():
    build.build()
    lib = B.load()
    assert lib.moe_trace_attach(None, 0, None, None) == B.MOE_ERR_NOT_BUILT
    assert "not in this build" in B.status_string(B.MOE_ERR_NOT_BUILT)
