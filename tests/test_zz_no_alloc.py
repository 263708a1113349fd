"""moe_dispatch_layout_noalloc: the dispatch layout for callers that cannot
allocate device memory (their device memory belongs to a framework's allocator
or a fixed memory plan, so they cannot hand the library a workspace).  It must
give exactly what moe_dispatch_layout gives with a workspace, call after call,
although every call reuses the library's one static scratch array.

This file is collected last on purpose, and it builds and loads the library
itself, so it passes both alone in a fresh process and after the other tests.
"""
import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200.inputs import make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    build.build()
    B.load()


def _problem(w, flags=0):
    return B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity, flags=flags)


def _outputs(buf, w):
    return {
        "status": buf.status.cpu().numpy().copy(),
        "expert_counts": buf.expert_counts.cpu().numpy().copy(),
        "expert_offsets": buf.expert_offsets.cpu().numpy().copy(),
        "meta": buf.meta.cpu().numpy().copy(),
        "row_src": buf.row_src.cpu().numpy()[:buf.rows].copy(),
        "pair_slot": buf.pair_slot.cpu().numpy()[:w.N].copy(),
        "drop_mask": buf.drop_mask.cpu().numpy()[:w.N].copy(),
    }


def _poisoned(prob):
    # poison the outputs so a skipped write cannot pass
    buf = B.Buffers(prob, quant=False)
    for t in (buf.expert_counts, buf.expert_offsets, buf.meta, buf.row_src, buf.pair_slot):
        t.fill_(-7)
    buf.drop_mask.fill_(9)
    buf.status.fill_(-1)
    return buf


def _noalloc(prob, ids, buf):
    B.moe_dispatch_layout_noalloc(prob, ids, buf.expert_counts, buf.expert_offsets, buf.meta,
                                  buf.row_src, buf.pair_slot, buf.drop_mask, buf.status)


def _run_both(w, flags=0):
    prob = _problem(w, flags)
    ids = torch.from_numpy(w.ids).cuda()
    ref = _poisoned(prob)
    B.moe_dispatch_layout(prob, ids, ref.expert_counts, ref.expert_offsets, ref.meta,
                          ref.row_src, ref.pair_slot, ref.drop_mask, ref.status, ref.workspace)
    got = _poisoned(prob)
    _noalloc(prob, ids, got)
    torch.cuda.synchronize()
    return _outputs(ref, w), _outputs(got, w)


def test_noalloc_layout_matches_workspace_layout_twice_in_a_row():
    # two calls in a row on different problems, then the first one again: each
    # call must see a clean scratch although the previous call used it
    for w in (make_workload("fp8_metric", with_expert_out=False, with_hidden=False),
              make_workload("decode_capacity", with_expert_out=False, with_hidden=False),
              make_workload("fp8_metric", with_expert_out=False, with_hidden=False)):
        ref, got = _run_both(w, flags=B.MOE_FLAG_CHECK_DUPLICATES)
        for key in ref:
            assert np.array_equal(ref[key], got[key]), (w.name, key)
        assert int(got["status"][0]) == 0


def test_noalloc_after_a_call_that_timed_out():
    """A call whose bounded waits run out (the test hook withholds the first
    scan tile's counts) still leaves the shared scratch usable: the next
    call matches the workspace path exactly."""
    from combine_topk_ids_scan_b200.inputs import Workload
    rng = np.random.default_rng(41)
    N, k, E = 3000, 4, 16                     # 12000 pairs: 3 scan tiles
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    w = Workload(name="stall", N=N, H=64, E=E, k=k, S=4, recv_capacity=N * k,
                 expert_capacity=0, ids=ids, gates=np.ones((N, k), np.float32),
                 hidden=np.zeros((N, 64), np.uint16), expert_out=None, global_scale=1.0, seed=0)
    prob = _problem(w, flags=B.MOE_FLAG_TEST_STALL_SCAN)
    buf = _poisoned(prob)
    _noalloc(prob, torch.from_numpy(ids).cuda(), buf)
    torch.cuda.synchronize()
    assert int(buf.status.cpu().numpy().view(np.uint32)[0]) & B.MOE_STATUS_TIMEOUT
    for _ in range(2):
        ref, got = _run_both(w)
        for key in ref:
            assert np.array_equal(ref[key], got[key]), key
        assert int(got["status"][0]) == 0


def test_noalloc_rejects_problems_beyond_the_scratch():
    # 8M pairs at E = 256 need more than 1 MiB of scan state
    prob = B.Problem(num_tokens=1 << 20, hidden=64, num_experts=256, top_k=8,
                     num_segments=8, recv_capacity=8 << 20)
    assert B.moe_workspace_bytes(prob) > B.MOE_NOALLOC_SCRATCH_BYTES
    buf = B.Buffers(prob, quant=False)
    ids = torch.zeros((1 << 20, 8), dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        _noalloc(prob, ids, buf)
    assert e.value.code == B.MOE_ERR_UNSUPPORTED_SHAPE
