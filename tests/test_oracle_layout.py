"""Pins for the oracle's dispatch layout (CPU only).

Independent formulations: numpy's stable argsort / bincount / cumsum, a
hand-worked example (tests/golden/layout_hand_example.txt), brute force over
every id matrix of tiny problems, and the invariants the NKI permute_a2av
reference states (displacements = exclusive cumsum of counts, the source map
is a permutation inside its segments, zero padding up to recv_capacity, the
dropless bound and its failure under duplicate ids).
"""
import itertools
import os

import numpy as np
import pytest

from combine_topk_ids_scan_b200.inputs import make_workload

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def numpy_layout(ids, E, S, H, C=0, Ce=0, pad=0):
    """Second formulation of the layout through numpy's stable sort."""
    N, k = ids.shape
    flat = ids.reshape(-1).astype(np.int64)
    valid = (flat >= 0) & (flat < E)
    pidx = np.nonzero(valid)[0]
    order = pidx[np.argsort(flat[pidx], kind="stable")]    # pairs, expert-major
    cnt = np.bincount(flat[pidx], minlength=E).astype(np.int64)
    first = np.concatenate([[0], np.cumsum(cnt)])          # start of each group
    rank = np.empty(flat.size, np.int64)
    rank[order] = np.arange(order.size) - first[flat[order]]
    slot = np.full(flat.size, -1, np.int64)
    drop = np.zeros(flat.size, np.uint8)
    if Ce > 0:
        rows = E * Ce
        keep = valid & (rank < Ce)
        slot[keep] = flat[keep] * Ce + rank[keep]
        drop[valid & ~keep] = 1
        counts = np.minimum(cnt, Ce)
        offsets = np.arange(E + 1) * Ce
    else:
        rows = C
        block = cnt if pad <= 1 else -(-cnt // pad) * pad     # counts rounded up
        start = np.concatenate([[0], np.cumsum(block)])
        pos = np.full(flat.size, -1, np.int64)
        pos[valid] = start[flat[valid]] + rank[valid]
        keep = valid & (pos < C)
        slot[keep] = pos[keep]
        drop[valid & ~keep] = 1
        counts = cnt
        offsets = start
    row_src = np.full(rows, -1, np.int64)
    row_src[slot[slot >= 0]] = np.nonzero(slot >= 0)[0] // k
    L = E // S
    if Ce > 0:
        seg_rows = counts.reshape(S, L).sum(axis=1)
    else:
        seg_rows = (offsets[1:] - offsets[:-1]).reshape(S, L).sum(axis=1)
    m0 = seg_rows * H
    m1 = (np.arange(S) * L * Ce * H) if Ce > 0 else np.concatenate([[0], np.cumsum(m0)[:-1]])
    meta = np.stack([m0, m1, m0, m1]).astype(np.uint32)
    return dict(expert_counts=counts, expert_offsets=offsets, pair_slot=slot.reshape(N, k),
                row_src=row_src, drop_mask=drop.reshape(N, k), meta=meta)


def check_equal(lay, ref):
    for key, want in ref.items():
        got = getattr(lay, key)
        assert np.array_equal(np.asarray(got).astype(np.int64).reshape(-1),
                              np.asarray(want).astype(np.int64).reshape(-1)), key


def test_hand_worked_example(orc):
    fx = {}
    for line in open(os.path.join(GOLDEN, "layout_hand_example.txt")):
        line = line.strip()
        if line and not line.startswith("#"):
            key, *vals = line.split()
            fx[key] = np.array([int(v) for v in vals])
    ids = fx["ids"].reshape(3, 2)
    lay = orc.layout(ids, 4, 2, 10, recv_capacity=8)
    assert lay.status == 0
    for key in ("expert_counts", "expert_offsets", "pair_slot", "row_src", "meta"):
        assert np.array_equal(getattr(lay, key).reshape(-1).astype(np.int64),
                              fx["packed." + key]), key
    lay = orc.layout(ids, 4, 2, 10, expert_capacity=2)
    assert lay.status == 0
    for key in ("expert_counts", "expert_offsets", "pair_slot", "row_src", "meta",
                "drop_mask"):
        assert np.array_equal(getattr(lay, key).reshape(-1).astype(np.int64),
                              fx["capacity." + key]), key
    lay = orc.layout(ids, 4, 2, 10, recv_capacity=16, expert_pad_multiple=4)
    assert lay.status == 0
    for key in ("expert_counts", "expert_offsets", "pair_slot", "row_src", "meta"):
        assert np.array_equal(getattr(lay, key).reshape(-1).astype(np.int64),
                              fx["pad4." + key]), key


@pytest.mark.parametrize("N,k,E,S", [(1, 1, 2, 1), (2, 2, 2, 2), (3, 2, 3, 1), (2, 3, 2, 1)])
def test_brute_force_all_id_matrices(orc, N, k, E, S):
    """Every ids matrix over {-1, 0..E-1} (masked ids and duplicates included)
    against the stable-sort formulation, in packed mode (ample and tight
    capacity) and capacity mode."""
    H = 3
    for flat in itertools.product(range(-1, E), repeat=N * k):
        ids = np.array(flat, np.int32).reshape(N, k)
        for C in (N * k, max(1, N * k - 2), N * k + 3):
            lay = orc.layout(ids, E, S, H, recv_capacity=C)
            ref = numpy_layout(ids, E, S, H, C=C)
            check_equal(lay, ref)
            overflow = int(((ids >= 0).sum()) > C)
            assert bool(lay.status & orc.STATUS_CAPACITY) == bool(overflow)
        for Ce in (1, 2):
            lay = orc.layout(ids, E, S, H, expert_capacity=Ce)
            check_equal(lay, numpy_layout(ids, E, S, H, Ce=Ce))
            assert lay.status == 0
        for pad, C in ((2, N * k * 2), (3, N * k + 2)):
            lay = orc.layout(ids, E, S, H, recv_capacity=C, expert_pad_multiple=pad)
            check_equal(lay, numpy_layout(ids, E, S, H, C=C, pad=pad))


def test_id_range_and_duplicates_status(orc):
    ids = np.array([[0, 5], [1, 1], [-1, -2]], np.int32)
    lay = orc.layout(ids, 4, 2, 8, recv_capacity=8, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status & orc.STATUS_ID_RANGE
    assert lay.status & orc.STATUS_DUP_ID
    # out-of-range ids (5, -2) are treated as masked: no row, not counted
    assert lay.pair_slot[0, 1] == -1 and lay.pair_slot[2, 1] == -1
    assert lay.expert_counts.sum() == 3
    lay = orc.layout(ids, 4, 2, 8, recv_capacity=8)          # no duplicate check
    assert not (lay.status & orc.STATUS_DUP_ID)


def test_id_equal_to_num_experts_is_out_of_range(orc):
    """Valid ids are [0, E): E itself is reported and treated as masked (no
    row, not counted, not a drop), in both modes."""
    ids = np.array([[4, 0], [3, 4], [2, 1]], np.int32)
    for kw in (dict(recv_capacity=8), dict(expert_capacity=2)):
        lay = orc.layout(ids, 4, 2, 8, **kw)
        assert lay.status == orc.STATUS_ID_RANGE
        assert lay.pair_slot[0, 0] == -1 and lay.pair_slot[1, 1] == -1
        assert lay.drop_mask.sum() == 0
        assert lay.expert_counts.tolist() == [1, 1, 1, 1]
        ref = numpy_layout(ids, 4, 2, 8, C=kw.get("recv_capacity", 0),
                           Ce=kw.get("expert_capacity", 0))
        check_equal(lay, ref)


@pytest.mark.parametrize("where", ["first", "middle", "last"])
def test_duplicate_check_reaches_every_token(orc, where):
    """A single token naming one expert twice is reported wherever it sits;
    without it the same matrix is clean."""
    N, k, E = 9, 3, 16
    ids = (np.arange(N * k, dtype=np.int32) % E).reshape(N, k)   # distinct per token
    lay = orc.layout(ids, E, 4, 8, recv_capacity=N * k, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == 0
    t = {"first": 0, "middle": N // 2, "last": N - 1}[where]
    ids[t, k - 1] = ids[t, 0]
    lay = orc.layout(ids, E, 4, 8, recv_capacity=N * k, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == orc.STATUS_DUP_ID


def test_duplicate_check_with_fewer_tokens_than_choices(orc):
    """One token, three choices, the duplicate in the last two."""
    ids = np.array([[2, 1, 1]], np.int32)
    lay = orc.layout(ids, 4, 2, 8, recv_capacity=3, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == orc.STATUS_DUP_ID


def test_duplicate_check_ignores_masked_and_out_of_range_ids(orc):
    """Reading: the duplicate check concerns experts a token is routed to, so
    repeated -1 (masked) entries are not duplicates, and repeated out-of-range
    ids are reported as out of range only."""
    ids = np.array([[-1, -1, 0], [2, 1, 3]], np.int32)
    lay = orc.layout(ids, 4, 2, 8, recv_capacity=6, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == 0
    ids = np.array([[4, 4, 0], [-2, -2, 1]], np.int32)
    lay = orc.layout(ids, 4, 2, 8, recv_capacity=6, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == orc.STATUS_ID_RANGE


@pytest.mark.parametrize("cfg", ["tiny", "mid_zipf", "nvfp4_hot", "balanced_static"])
def test_packed_invariants_on_workloads(orc, cfg):
    w = make_workload(cfg, n_tokens=2048 if cfg != "tiny" else None,
                      with_expert_out=False, with_hidden=False)
    C = w.recv_capacity
    lay = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status == 0
    check_equal(lay, numpy_layout(w.ids, w.E, w.S, w.H, C=C))
    # counts sum to N * top_k (no masked ids in these workloads)
    assert lay.expert_counts.sum() == w.N * w.k
    # displacements are the exclusive cumsum of counts
    assert np.array_equal(lay.expert_offsets[1:] - lay.expert_offsets[:-1], lay.expert_counts)
    m = lay.meta.astype(np.int64)
    assert np.array_equal(m[1], np.concatenate([[0], np.cumsum(m[0])[:-1]]))
    assert m[1, -1] + m[0, -1] == w.N * w.k * w.H
    assert np.array_equal(m[2], m[0]) and np.array_equal(m[3], m[1])
    # pair_slot <-> row_src is a bijection between routed pairs and rows
    slots = lay.pair_slot.reshape(-1)
    assert np.array_equal(np.sort(slots), np.arange(w.N * w.k))
    assert np.array_equal(lay.row_src[slots], np.arange(w.N * w.k) // w.k)
    # expert e's rows are [off[e], off[e+1]); sources strictly increase in them
    for e in range(w.E):
        seg = lay.row_src[lay.expert_offsets[e]:lay.expert_offsets[e + 1]]
        assert np.all(np.diff(seg) > 0)
        assert np.all((w.ids[seg] == e).any(axis=1))
    # the dropless bound: each destination segment receives <= N*min(k, L)
    L = w.E // w.S
    seg_rows = lay.expert_counts.reshape(w.S, L).sum(axis=1)
    assert np.all(seg_rows <= w.N * min(w.k, L))


def test_zero_padding_rows(orc):
    rng = np.random.default_rng(7)
    ids = rng.integers(-1, 8, size=(100, 3)).astype(np.int32)
    C = 400
    lay = orc.layout(ids, 8, 4, 16, recv_capacity=C)
    total = int((ids >= 0).sum())
    assert total < C
    assert np.all(lay.row_src[total:] == -1) and np.all(lay.row_src[:total] >= 0)


def test_dropless_bound_fails_with_duplicates(orc):
    """L = 1 and every token routed to [0, 0]: segment 0 receives 2N rows,
    more than N * min(k, L) = N, as the recv_capacity note predicts."""
    N = 50
    ids = np.zeros((N, 2), np.int32)
    lay = orc.layout(ids, 4, 4, 8, recv_capacity=2 * N, flags=orc.FLAG_CHECK_DUPLICATES)
    assert lay.status & orc.STATUS_DUP_ID
    seg0 = lay.meta[0, 0] // 8
    assert seg0 == 2 * N > N * min(2, 1)
    # with recv_capacity at the (now wrong) bound the overflow is reported
    lay = orc.layout(ids, 4, 4, 8, recv_capacity=N)
    assert lay.status & orc.STATUS_CAPACITY
    assert (lay.pair_slot >= 0).sum() == N and lay.drop_mask.sum() == N
    assert lay.expert_counts[0] == 2 * N          # counts stay the true counts


def test_capacity_mode_decode_workload(orc):
    w = make_workload("decode_capacity", with_expert_out=False, with_hidden=False)
    assert w.expert_capacity == 5
    lay = orc.layout(w.ids, w.E, w.S, w.H, expert_capacity=w.expert_capacity)
    check_equal(lay, numpy_layout(w.ids, w.E, w.S, w.H, Ce=w.expert_capacity))
    cnt = np.bincount(w.ids.reshape(-1), minlength=w.E)
    kept = (lay.pair_slot >= 0).sum()
    assert kept + lay.drop_mask.sum() == w.N * w.k
    assert np.array_equal(lay.expert_counts, np.minimum(cnt, 5))
    # kept pairs of each expert are its first Ce pairs in (token, k) order
    flat = w.ids.reshape(-1)
    for e in range(w.E):
        p = np.nonzero(flat == e)[0]
        s = lay.pair_slot.reshape(-1)[p]
        assert np.array_equal(s[:5], e * 5 + np.arange(min(5, p.size)))
        assert np.all(s[5:] == -1)
    m = lay.meta.astype(np.int64)
    assert np.array_equal(m[1], np.arange(w.S) * (w.E // w.S) * 5 * w.H)


@pytest.mark.parametrize("pad", [1, 4, 16, 128])
def test_expert_padding_invariants(orc, pad):
    """Every expert block starts at a multiple of pad and holds the expert's
    rows first, then padding; nothing else changes."""
    w = make_workload("mid_zipf", n_tokens=1024, with_expert_out=False, with_hidden=False)
    C = w.N * w.k + w.E * pad
    lay = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C, expert_pad_multiple=pad)
    assert lay.status == 0
    check_equal(lay, numpy_layout(w.ids, w.E, w.S, w.H, C=C, pad=pad))
    off = lay.expert_offsets.astype(np.int64)
    assert np.all(off % max(pad, 1) == 0)
    for e in range(w.E):
        n = lay.expert_counts[e]
        blk = lay.row_src[off[e]:off[e + 1]]
        assert np.all(blk[:n] >= 0) and np.all(blk[n:] == -1)
        assert off[e + 1] - off[e] == -(-n // max(pad, 1)) * max(pad, 1)
    base = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C)
    # the source order inside each expert is the unpadded one
    for e in range(w.E):
        n = lay.expert_counts[e]
        assert np.array_equal(lay.row_src[off[e]:off[e] + n],
                              base.row_src[base.expert_offsets[e]:base.expert_offsets[e] + n])
