"""Host-side logic of the benchmark, including its multi-rank path, run as
world_size-2 gloo process groups on the CPU."""
import os
import socket

import torch.distributed as dist
import torch.multiprocessing as mp

import bench
from combine_topk_ids_scan_b200.inputs import make_workload


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _worker(rank, world, port, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        out = bench.max_over_ranks([1.0 + rank, 10.0 - rank, 0.5 * rank], "cpu", world)
        q.put((rank, out))
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_gloo_world2():
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q)) for r in range(2)]
    for p in procs:
        p.start()
    res = dict(q.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(2):
        assert res[r] == [2.0, 10.0, 0.5]


def test_rank_batches_are_independent_replicas():
    assert bench.seed_for_rank(0) is None
    seeds = {bench.seed_for_rank(r) for r in range(1, 8)}
    assert len(seeds) == 7
    a = make_workload("tiny", seed=bench.seed_for_rank(1), with_expert_out=False)
    b = make_workload("tiny", with_expert_out=False)
    assert a.ids.shape == b.ids.shape and (a.ids != b.ids).any()


def test_reference_arm_nonzero_rank_does_nothing(capsys):
    class A:
        steps, warmup = 5, 3
    assert bench.run_reference(A(), rank=1, world=2) == 0
    assert capsys.readouterr().out == ""


def test_algorithmic_bytes_metric_workload():
    w = make_workload("fp8_metric", with_expert_out=False, with_hidden=False)
    nb = bench.algorithmic_bytes(w, total_rows=w.N * w.k)
    N, H, C = 8192, 7168, 65536
    # hidden read once, every output row written once (plus the small maps)
    assert nb["permute_bf16"] == 2 * N * H + 2 * C * H + 4 * C + 4 * C
    assert nb["combine"] == 2 * C * H + 8 * C + 2 * N * H
    assert abs(nb["permute_fp8"] - (2 * N * H + C * H + 4 * C * 56)) < 1e6
