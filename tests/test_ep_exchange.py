"""Expert-parallel exchange (combine_topk_ids_scan_b200/ep.py) as
world-size-2 and world-size-4 gloo process groups on the CPU.

Every rank routes its own seeded tokens; the local layout and permutes come
from the oracle (this test's input), the exchange from the library's ep
module.  Each rank recomputes every other rank's oracle result from the
known seeds and checks: the receive counts and displacements written into
meta rows 2-3 (the [4, EP] table of permute_a2av), the per-expert counts of
every source, the received rows (bf16 rows, FP8 code and scale rows) equal
the concatenation over source ranks of their segment for this rank, and the
combine exchange returns every row to the position it left.
"""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from combine_topk_ids_scan_b200 import ep


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_problem(r, world, mode):
    """Seeded tokens of rank r: N tokens, top-k distinct experts."""
    rng = np.random.default_rng(500 + r)
    N, H, L, k = 40 + 7 * r, 256, 3, 2
    E = L * world
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    ids[rng.random((N, k)) < 0.1] = -1                       # some masked pairs
    hidden = (rng.standard_normal((N, H)).astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)
    Ce = 4 if mode == "capacity" else 0
    C = 0 if Ce else N * k + 5
    pad = 4 if mode == "padded" else 0
    if pad:
        C = N * k + E * (pad - 1)
    return dict(ids=ids, hidden=hidden, N=N, H=H, E=E, k=k, S=world, C=C, Ce=Ce, pad=pad)


def _oracle_dispatch(orc, p):
    lay = orc.layout(p["ids"], p["E"], p["S"], p["H"], recv_capacity=p["C"],
                     expert_capacity=p["Ce"], expert_pad_multiple=p["pad"])
    out = orc.permute_bf16(p["hidden"], lay.row_src)
    q8, s8 = orc.permute_fp8(p["hidden"], lay.row_src)
    return lay, out, q8, s8


def _segment_rows(lay, p, s):
    """Rows of segment s of rank p's dispatch output (the rows shipped to s)."""
    L = p["E"] // p["S"]
    if p["Ce"]:
        return np.arange(s * L * p["Ce"], (s + 1) * L * p["Ce"])
    lo, hi = lay.expert_offsets[s * L], lay.expert_offsets[(s + 1) * L]
    return np.arange(lo, hi)


def _worker(rank, world, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        import oracle as orc
        probs = [_rank_problem(r, world, mode) for r in range(world)]
        refs = [_oracle_dispatch(orc, p) for p in probs]
        p = probs[rank]
        lay, out, q8, s8 = refs[rank]
        meta = torch.from_numpy(lay.meta.view(np.int32).copy())
        route = ep.exchange_counts(meta, p["H"], p["E"], expert_capacity=p["Ce"])
        # receive counts / displacements (elements) in meta rows 2-3
        recv_rows = [len(_segment_rows(refs[s][0], probs[s], rank)) for s in range(world)]
        got2 = meta[2].numpy().view(np.uint32).astype(np.int64)
        got3 = meta[3].numpy().view(np.uint32).astype(np.int64)
        assert list(got2) == [r * p["H"] for r in recv_rows], (got2, recv_rows)
        assert list(got3) == list(np.cumsum([0] + recv_rows[:-1]) * p["H"])
        assert route.recv_rows == recv_rows
        # put offsets for the fused send: where this rank's block starts in
        # every receiver's buffer (the receiver's displacement of this source)
        po = ep.put_offsets(route)
        want_po = [sum(len(_segment_rows(refs[s][0], probs[s], d)) for s in range(rank))
                   for d in range(world)]
        assert po == want_po, (po, want_po)
        # per-expert counts of every source for this rank's experts
        L = p["E"] // world
        ec = ep.exchange_expert_counts(torch.from_numpy(lay.expert_counts.copy()))
        want_ec = np.stack([refs[s][0].expert_counts[rank * L:(rank + 1) * L] for s in range(world)])
        assert np.array_equal(ec.numpy(), want_ec)
        # payload rows: bf16 rows, FP8 codes and scales
        for mine, j in ((out, 1), (q8, 2), (s8, 3)):
            recv = ep.dispatch_exchange(torch.from_numpy(mine.copy()), route)
            want = np.concatenate([refs[s][j][_segment_rows(refs[s][0], probs[s], rank)]
                                   for s in range(world)])
            assert np.array_equal(recv.numpy(), want), j
        # combine route: identity experts send the rows straight back
        recv = ep.dispatch_exchange(torch.from_numpy(out.copy()), route)
        back = ep.combine_exchange(recv, route)
        sent = route.send_total
        assert np.array_equal(back.numpy()[:sent], out[:sent])
        # argument errors are raised before any collective (every rank raises)
        bad = torch.zeros((4, world + 1), dtype=torch.int32)
        try:
            ep.exchange_counts(bad, p["H"], p["E"])
            raise AssertionError("segments != ranks accepted")
        except ValueError:
            pass
        one_each = ep.Route(send_rows=[1] * world, recv_rows=[1] * world)
        for call, rows in ((ep.dispatch_exchange, world - 1), (ep.combine_exchange, world + 1)):
            try:
                call(torch.zeros((rows, 4)), one_each)
                raise AssertionError(f"{call.__name__}: wrong row count accepted")
            except ValueError:
                pass
        try:
            ep.combine_exchange(torch.zeros((world, 4)), one_each,
                                out=torch.zeros((world, 4), dtype=torch.float64))
            raise AssertionError("combine_exchange: out of another dtype accepted")
        except ValueError:
            pass
        q.put((rank, "ok"))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 4])
@pytest.mark.parametrize("mode", ["packed", "padded", "capacity"])
def test_ep_exchange_gloo(world, mode):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
    assert all(v == "ok" for v in res.values()), res
