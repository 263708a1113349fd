"""The dispatch fused with the expert-parallel send, run by two and three
ranks: as many processes on one GPU, a gloo group for the counts, offsets and barriers,
each rank's receive buffers mapped into the other process with CUDA IPC
(torch's CUDA tensor sharing).

Every rank routes its own seeded tokens through the library's layout,
exchanges counts (ep.exchange_counts) and put offsets (ep.put_offsets),
then stores its segments straight into the owners' receive buffers with
moe_permute_to_peers, moe_permute_quant_fp8_to_peers and
moe_permute_quant_nvfp4_to_peers.  After a device synchronisation and a
barrier, with identity experts (the received bf16 rows are the expert
outputs), every rank combines with moe_combine_from_peers, reading its rows
back from the owners' buffers, and checks the result against the oracle's
combine of its own dispatch; each rank then checks its own receive buffers,
every row, code and scale, against the concatenation over source ranks of
the oracle's dispatch segments for it, and that no row past them was
touched.  The kernels never
wait on another process (completion is the host barrier), so the two ranks
sharing one GPU cannot deadlock; across GPUs the same stores go over NVLink.

A last case runs the ep module's host-level route on the NCCL backend with
CUDA tensors, with one rank (NCCL takes one rank per GPU).
"""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

pytestmark = pytest.mark.gpu

def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _shared_gpu_allowed() -> bool:
    """Several processes may hold a context on device 0 (compute mode
    Default); read through NVML, changing nothing."""
    try:
        import pynvml
        pynvml.nvmlInit()
        try:
            h = pynvml.nvmlDeviceGetHandleByIndex(0)
            return pynvml.nvmlDeviceGetComputeMode(h) == pynvml.NVML_COMPUTEMODE_DEFAULT
        finally:
            pynvml.nvmlShutdown()
    except Exception:
        return True   # no NVML: let the test find out


def _rank_problem(r, mode, world=1):
    rng = np.random.default_rng(900 + r)
    N, H, L, k = 300 + 37 * r, 384, 4, 3
    E = L * world
    ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
    ids[rng.random((N, k)) < 0.05] = -1
    hidden = (rng.standard_normal((N, H)).astype(np.float32).view(np.uint32) >> 16).astype(
        np.uint16)
    amax = float(np.abs((hidden.astype(np.uint32) << 16).view(np.float32)).max())
    Ce = 80 if mode == "capacity" else 0
    pad = 8 if mode == "padded" else 0
    C = 0 if Ce else (N * k + E * (pad - 1) if pad else N * k + 3)
    return dict(ids=ids, hidden=hidden, N=N, H=H, E=E, k=k, C=C, Ce=Ce, pad=pad,
                gs=float(np.float32(amax) / np.float32(2688.0)))


def _segment_rows(lay, p, s, world):
    L = p["E"] // world
    if p["Ce"]:
        return np.arange(s * L * p["Ce"], (s + 1) * L * p["Ce"])
    return np.arange(lay.expert_offsets[s * L], lay.expert_offsets[(s + 1) * L])


def _worker(rank, world, port, mode, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    # a short timeout: a rank that fails makes the other's next barrier fail
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    keep = []
    try:
        from torch.multiprocessing.reductions import reduce_tensor

        import oracle as orc
        from combine_topk_ids_scan_b200 import binding as B
        from combine_topk_ids_scan_b200 import ep
        torch.cuda.set_device(0)
        B.load()
        probs = [_rank_problem(r, mode, world) for r in range(world)]
        refs = []
        for p in probs:
            lay = orc.layout(p["ids"], p["E"], world, p["H"], recv_capacity=p["C"],
                             expert_capacity=p["Ce"], expert_pad_multiple=p["pad"])
            q8, s8 = orc.permute_fp8(p["hidden"], lay.row_src)
            q4, s4 = orc.permute_nvfp4(p["hidden"], lay.row_src, p["gs"])
            refs.append((lay, orc.permute_bf16(p["hidden"], lay.row_src), q8, s8.view(np.uint32),
                         q4, s4))
        p = probs[rank]
        H = p["H"]
        prob = B.Problem(num_tokens=p["N"], hidden=H, num_experts=p["E"], top_k=p["k"],
                         num_segments=world, recv_capacity=p["C"], expert_capacity=p["Ce"],
                         expert_pad_multiple=p["pad"])
        buf = B.Buffers(prob, quant=False)
        hid = torch.from_numpy(p["hidden"].view(np.int16)).cuda().view(torch.bfloat16)
        B.layout(prob, torch.from_numpy(p["ids"]).cuda(), buf)
        torch.cuda.synchronize()
        assert int(buf.status.item()) == refs[rank][0].status
        meta_host = buf.meta.cpu()
        route = ep.exchange_counts(meta_host, H, p["E"], expert_capacity=p["Ce"])
        put = torch.tensor(ep.put_offsets(route), dtype=torch.int64, device="cuda")
        # this rank's receive buffers (two spare rows at the end), poisoned
        n = route.recv_total + 2
        mine = [torch.full((n, H), 0x7FC1, dtype=torch.int16, device="cuda"),
                torch.full((n, H), 0xA5, dtype=torch.uint8, device="cuda"),
                torch.full((n, H // 128), 0x7FA5A5A5, dtype=torch.int32, device="cuda"),
                torch.full((n, H // 2), 0xA5, dtype=torch.uint8, device="cuda"),
                torch.full((n, H // 16), 0xA5, dtype=torch.uint8, device="cuda")]
        torch.cuda.synchronize()
        # share them: every rank maps every other rank's buffers
        handles = [None] * world
        dist.all_gather_object(handles, [reduce_tensor(t) for t in mine])
        bufs = []
        for r in range(world):
            if r == rank:
                bufs.append(mine)
            else:
                mapped = [fn(*args) for fn, args in handles[r]]
                keep.extend(mapped)
                bufs.append(mapped)

        def ptrs(i):
            return torch.tensor([bufs[r][i].data_ptr() for r in range(world)],
                                dtype=torch.int64, device="cuda")

        gs = torch.tensor([p["gs"]], dtype=torch.float32, device="cuda")
        B.moe_permute_to_peers(prob, hid, buf.row_src, buf.pair_slot, buf.meta, ptrs(0), put)
        B.moe_permute_quant_fp8_to_peers(prob, hid, buf.row_src, buf.pair_slot, buf.meta,
                                         ptrs(1), ptrs(2), put)
        B.moe_permute_quant_nvfp4_to_peers(prob, hid, buf.row_src, buf.pair_slot, buf.meta, gs,
                                           ptrs(3), ptrs(4), put)
        torch.cuda.synchronize()
        dist.barrier()
        # identity experts: each rank's received bf16 rows are its expert
        # outputs; every rank combines reading its rows back from the owners
        gates = np.random.default_rng(1300 + rank).random((p["N"], p["k"])).astype(np.float32)
        y = torch.empty((p["N"], H), dtype=torch.bfloat16, device="cuda")
        B.moe_combine_from_peers(prob, ptrs(0), put, buf.meta, torch.from_numpy(gates).cuda(),
                                 buf.pair_slot, y)
        torch.cuda.synchronize()
        want_y = orc.combine(refs[rank][1], gates, refs[rank][0].pair_slot)
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want_y), mode
        dist.barrier()
        # every row this rank received, from every source, in source order
        total = route.recv_total
        got = [t.cpu().numpy() for t in mine]
        got[0] = got[0].view(np.uint16)
        got[2] = got[2].view(np.uint32)
        for i, j in ((0, 1), (1, 2), (2, 3), (3, 4), (4, 5)):
            want = np.concatenate([refs[s][j][_segment_rows(refs[s][0], probs[s], rank, world)]
                                   for s in range(world)])
            assert want.shape[0] == total
            assert np.array_equal(got[i][:total], want), (mode, i)
        assert np.all(got[0][total:] == 0x7FC1) and np.all(got[1][total:] == 0xA5)
        assert np.all(got[2][total:] == 0x7FA5A5A5) and np.all(got[4][total:] == 0xA5)
        # close the mappings of the other rank's buffers, then wait for it to
        # do the same before any buffer is freed
        keep.clear()
        torch.cuda.synchronize()
        dist.barrier()
        q.put((rank, "ok"))
    except Exception as e:  # report to the parent instead of hanging it
        q.put((rank, repr(e)))
    finally:
        keep.clear()
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("mode", ["packed", "padded", "capacity"])
def test_fused_send_between_processes(orc, mode, world):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    if not _shared_gpu_allowed():
        pytest.skip("the GPU's compute mode admits one process at a time")
    from combine_topk_ids_scan_b200 import build
    build.build()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, mode, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=300) for _ in procs)
    for p in procs:
        p.join(timeout=120)
    assert all(v == "ok" for v in res.values()), res


def _nccl_single(port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    try:
        torch.cuda.set_device(0)
        dist.init_process_group("nccl", rank=0, world_size=1,
                                timeout=datetime.timedelta(seconds=120))
        import oracle as orc
        from combine_topk_ids_scan_b200 import binding as B
        from combine_topk_ids_scan_b200 import ep
        B.load()
        p = _rank_problem(0, "packed", 1)
        N, H, E, k = p["N"], p["H"], p["E"], p["k"]
        prob = B.Problem(num_tokens=N, hidden=H, num_experts=E, top_k=k, num_segments=1,
                         recv_capacity=p["C"])
        buf = B.Buffers(prob, quant=False)
        hid = torch.from_numpy(p["hidden"].view(np.int16)).cuda().view(torch.bfloat16)
        B.layout(prob, torch.from_numpy(p["ids"]).cuda(), buf)
        B.moe_permute(prob, hid, buf.row_src, buf.pair_slot, buf.out)
        # the counts all-to-all and the payload route on NCCL, CUDA tensors
        route = ep.exchange_counts(buf.meta, H, E)
        recv = ep.dispatch_exchange(buf.out, route)
        gates = torch.from_numpy(
            np.full((N, k), 1.0 / k, np.float32)).cuda()
        back = ep.combine_exchange(recv, route, out=torch.zeros_like(buf.out))
        y = torch.empty((N, H), dtype=torch.bfloat16, device="cuda")
        B.moe_combine(prob, back, gates, buf.pair_slot, y)
        torch.cuda.synchronize()
        lay = orc.layout(p["ids"], E, 1, H, recv_capacity=p["C"])
        out = orc.permute_bf16(p["hidden"], lay.row_src)
        assert np.array_equal(recv.view(torch.int16).cpu().numpy().view(np.uint16),
                              out[:route.recv_total])
        assert np.array_equal(buf.meta.cpu().numpy()[2:], buf.meta.cpu().numpy()[:2])
        want = orc.combine(out, np.full((N, k), 1.0 / k, np.float32), lay.pair_slot)
        assert np.array_equal(y.view(torch.int16).cpu().numpy().view(np.uint16), want)
        q.put("ok")
    except Exception as e:  # report to the parent instead of hanging it
        q.put(repr(e))
    finally:
        if dist.is_initialized():
            dist.destroy_process_group()


def test_ep_module_on_nccl_with_one_rank(orc):
    """The ep module's collectives on the NCCL backend with CUDA tensors (one
    rank: the counts all-to-all is a self exchange, the payload route a
    local copy): a dispatch, its exchange there and back, and the combine
    of the returned rows match the oracle."""
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    proc = ctx.Process(target=_nccl_single, args=(_free_port(), q))
    proc.start()
    res = q.get(timeout=300)
    proc.join(timeout=120)
    assert res == "ok", res
