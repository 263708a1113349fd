"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle.

Integer, index and byte outputs must match bit for bit; the combine is
computed with the same fp32 fused multiply-adds in the same order, so it must
match bit for bit as well (which is inside the 1-bf16-ulp contract; the
contract bound itself is checked separately against a float64 sum).
"""
import zlib

import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200.inputs import Workload, make_workload, normal_bf16, softmax_gates
from gpu_util import (GpuRun, bf16_np, par_rows, poison, poison_buffers, poisoned_empty,
                      problem_of, to_dev_bf16)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    build.build()
    B.load()


def custom(N, H, E, k, S, C=None, Ce=0, ids=None, seed=0, p_mask=0.0, p_bad=0.0,
           distinct=True, with_out=True):
    ss = np.random.SeedSequence(seed)
    s_ids, s_g, s_h, s_o = ss.spawn(4)
    rng = np.random.Generator(np.random.PCG64(s_ids))
    if ids is None:
        if distinct and k <= E:
            ids = np.argsort(rng.random((N, E)), axis=1)[:, :k].astype(np.int32)
        else:
            ids = rng.integers(0, E, size=(N, k)).astype(np.int32)
        m = rng.random((N, k))
        ids[m < p_mask] = -1
        bad = rng.random((N, k)) < p_bad
        ids[bad] = rng.choice([-7, E, E + 3, -2], size=int(bad.sum()))
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    if C is None:
        C = N * k
    rows = E * Ce if Ce > 0 else C
    hidden = normal_bf16(s_h, N, H) if N > 0 else np.zeros((0, H), np.uint16)
    hv = (hidden.astype(np.uint32) << 16).view(np.float32)
    amax = float(np.abs(hv).max()) if hv.size else 0.0
    gs = float(np.float32(amax) / np.float32(2688.0)) if amax > 0 else 1.0
    gates = softmax_gates(np.random.Generator(np.random.PCG64(s_g)), N, k)
    X = normal_bf16(s_o, rows, H) if with_out else None
    return Workload(name="custom", N=N, H=H, E=E, k=k, S=S,
                    recv_capacity=0 if Ce > 0 else C, expert_capacity=Ce, ids=ids,
                    gates=gates, hidden=hidden, expert_out=X, global_scale=gs, seed=seed)


def oracle_layout(orc, w, flags=0, pad=0):
    return orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=w.recv_capacity,
                      expert_capacity=w.expert_capacity, flags=flags,
                      expert_pad_multiple=pad)


def assert_layout(run, ref):
    assert run.status == ref.status, (hex(run.status), hex(ref.status))
    for key in ("expert_counts", "expert_offsets", "meta", "row_src", "pair_slot", "drop_mask"):
        got, want = getattr(run, key), getattr(ref, key)
        assert np.array_equal(np.asarray(got).reshape(-1).astype(np.int64),
                              np.asarray(want).reshape(-1).astype(np.int64)), key


def assert_all_outputs(orc, w, run, ref):
    """Compare every payload row, scale and combined token with the oracle
    (the oracle runs over row / token chunks in threads: rows and tokens are
    independent)."""
    row_src = ref.row_src
    R = row_src.size
    want = par_rows(lambda rs: orc.permute_bf16(w.hidden, rs), R, row_src)
    assert np.array_equal(run.out, want), "bf16 permute"
    if run.has_fp8:
        q, s = par_rows(lambda rs: orc.permute_fp8(w.hidden, rs), R, row_src)
        assert np.array_equal(run.q8, q), "fp8 codes"
        assert np.array_equal(run.s8.view(np.uint32), s.view(np.uint32)), "fp8 scales"
    if run.has_fp4:
        swz = run.swizzled

        def same_scales(got, want_linear):
            if not swz:
                return np.array_equal(got, want_linear)
            if R == 0:                      # nothing is written; the buffer is one byte
                return True
            want = orc.swizzle_scales(want_linear).reshape(-1)
            return got.size == want.size and np.array_equal(got, want)

        q, s = par_rows(lambda rs: orc.permute_nvfp4(w.hidden, rs, w.global_scale), R, row_src)
        assert np.array_equal(run.q4, q), "nvfp4 codes"
        assert same_scales(run.s4, s), "nvfp4 scales"
        q, s = par_rows(lambda rs: orc.permute_mxfp4(w.hidden, rs), R, row_src)
        assert np.array_equal(run.qmx, q), "mxfp4 codes"
        assert same_scales(run.smx, s), "mxfp4 scales"
    if run.y is not None:
        y = par_rows(lambda g, ps: orc.combine(w.expert_out, g, ps), w.N, w.gates,
                     ref.pair_slot)
        assert np.array_equal(run.y, y), "combine"


# ------------------------------------------------------------ the workloads
@pytest.mark.parametrize("cfg", ["tiny", "mid_zipf", "decode_capacity"])
def test_workload_full_parity(orc, cfg):
    w = make_workload(cfg)
    run = GpuRun(w)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)


@pytest.mark.parametrize("cfg", ["fp8_metric", "nvfp4_hot", "balanced_static"])
def test_full_size_workload_parity(orc, cfg):
    """Full sizes, the launch configuration the benchmark times: every
    output row, scale and combined token compared with the oracle."""
    w = make_workload(cfg)
    run = GpuRun(w)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)


def test_identity_expert_round_trip_gpu(orc):
    w = make_workload("tiny")
    run = GpuRun(w, quant=False, combine=False)
    prob = problem_of(w)
    gates = torch.from_numpy(w.gates).cuda()
    y = poisoned_empty((w.N, w.H), torch.bfloat16)
    B.moe_combine(prob, run.buf.out, gates, run.buf.pair_slot, y)
    assert np.array_equal(bf16_np(y), w.hidden)


def test_combine_within_contract_of_exact_sum(orc):
    """The spec contract: <= 1 bf16 ulp of the exact weighted sum (plus
    the fp32 accumulation error bound)."""
    w = make_workload("mid_zipf", n_tokens=512)
    run = GpuRun(w, quant=False)
    xf = (w.expert_out.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    exact = np.zeros((w.N, w.H))
    mag = np.zeros((w.N, w.H))
    for j in range(w.k):
        s = run.pair_slot[:, j]
        term = w.gates[:, j:j + 1].astype(np.float64) * xf[s]
        exact += term
        mag += np.abs(term)
    got = (run.y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0**-126))) - 7)
    assert np.all(np.abs(got - exact) <= ulp + w.k * 2.0**-23 * mag)


# ------------------------------------------------------------ edge cases
EDGE = {
    "ragged_masked_badids": dict(N=3001, H=384, E=40, k=3, S=5, p_mask=0.1, p_bad=0.02),
    "packed_overflow": dict(N=700, H=256, E=16, k=4, S=4, C=1900),
    "padding_large": dict(N=300, H=128, E=8, k=2, S=2, C=1500, p_mask=0.3),
    "all_masked": dict(N=64, H=128, E=4, k=2, S=1, C=40, p_mask=1.1),
    "k1": dict(N=5000, H=96, E=7, k=1, S=7),
    "k16": dict(N=1300, H=256, E=64, k=16, S=16),
    "E1": dict(N=999, H=64, E=1, k=1, S=1),
    "E2048_S2048": dict(N=2048, H=32, E=2048, k=8, S=2048),
    "H65536": dict(N=40, H=65536, E=8, k=2, S=2, p_mask=0.1),
    "duplicates": dict(N=1000, H=128, E=6, k=4, S=3, distinct=False),
    "capacity_drops": dict(N=900, H=256, E=32, k=4, S=8, Ce=3),
    "capacity_masked": dict(N=333, H=160, E=12, k=3, S=4, Ce=40, p_mask=0.2, p_bad=0.01),
}


# the three layout kernels: chosen by size (the cluster kernel for every
# case here), the one-launch look-back kernel, the scan + emit kernels
LAYOUT_PATHS = {"auto": 0, "lookback": B.MOE_FLAG_LAYOUT_LOOKBACK,
                "two_pass": B.MOE_FLAG_LAYOUT_TWO_PASS}


@pytest.mark.parametrize("path", sorted(LAYOUT_PATHS))
@pytest.mark.parametrize("name", sorted(EDGE))
def test_edge_case_parity(orc, name, path):
    spec = dict(EDGE[name])
    w = custom(seed=zlib.crc32(name.encode()) % 1000, **spec)
    flags = B.MOE_FLAG_CHECK_DUPLICATES | LAYOUT_PATHS[path]
    run = GpuRun(w, flags=flags)
    ref = oracle_layout(orc, w, flags=orc.FLAG_CHECK_DUPLICATES)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)


def test_empty_problem(orc):
    w = custom(N=0, H=128, E=8, k=2, S=2, C=16)
    run = GpuRun(w)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    assert np.all(run.out == 0) and np.all(run.q8 == 0) and np.all(run.s4 == 0)


def test_many_tiles_multi_wave_scan(orc):
    """4M pairs = 1024 scan tiles, more than one wave of CTAs (the two-kernel
    path): the look-back chain crosses waves."""
    N, k, E = 262144, 16, 64
    rng = np.random.default_rng(5)
    ids = rng.integers(0, E, size=(N, k)).astype(np.int32)
    w = custom(N=N, H=8, E=E, k=k, S=4, ids=ids, with_out=False)
    run = GpuRun(w, quant=False, combine=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)


def test_workspace_reuse_across_problems(orc):
    """The layout leaves its workspace zeroed, so one buffer serves a
    sequence of different problems."""
    ws = torch.zeros(1 << 20, dtype=torch.uint8, device="cuda")
    for i, spec in enumerate([dict(N=5000, H=64, E=32, k=4, S=4),
                              dict(N=700, H=64, E=256, k=8, S=8),
                              dict(N=9000, H=64, E=5, k=2, S=5, p_mask=0.2)]):
        w = custom(seed=100 + i, with_out=False, **spec)
        prob = problem_of(w)
        assert B.moe_workspace_bytes(prob) <= ws.numel()
        buf = poison_buffers(B.Buffers(prob, quant=False))
        buf.workspace = ws
        for _ in range(2):
            B.layout(prob, torch.from_numpy(w.ids).cuda(), buf)
            torch.cuda.synchronize()
            ref = oracle_layout(orc, w)
            assert np.array_equal(buf.pair_slot.cpu().numpy()[:w.N], ref.pair_slot)
            assert np.array_equal(buf.row_src.cpu().numpy()[:buf.rows], ref.row_src)
        # every word the call used is back at zero
        assert int(ws.count_nonzero()) == 0


@pytest.mark.parametrize("two_pass", [False, True], ids=["fused", "two_pass"])
def test_scan_wait_times_out_with_status(orc, two_pass):
    """The test hook withholds the first tile's counts: every later tile's
    bounded wait runs out (about a second), the kernels finish, the status
    word reports MOE_STATUS_TIMEOUT and the device stays usable.  The
    workspace is returned to zero even then (in the one-launch kernel the
    blocks without a tile also give up their grid-wide wait, while the late
    tiles are still publishing), so the same workspace serves the next call."""
    w = custom(N=3000, H=64, E=16, k=4, S=4, with_out=False)   # 12000 pairs, 3 tiles
    prob = problem_of(w, flags=B.MOE_FLAG_TEST_STALL_SCAN |
                      (B.MOE_FLAG_LAYOUT_TWO_PASS if two_pass else 0))
    ids = torch.from_numpy(w.ids).cuda()
    buf = poison_buffers(B.Buffers(prob, quant=False))
    ws = buf.workspace
    B.layout(prob, ids, buf)
    torch.cuda.synchronize()
    assert int(buf.status.cpu().numpy().view(np.uint32)[0]) & B.MOE_STATUS_TIMEOUT
    assert int(ws.count_nonzero()) == 0
    # the context is intact: a normal call on the same workspace is exact
    prob = problem_of(w, flags=B.MOE_FLAG_LAYOUT_TWO_PASS if two_pass else 0)
    buf = poison_buffers(B.Buffers(prob, quant=False))
    buf.workspace = ws
    B.layout(prob, ids, buf)
    torch.cuda.synchronize()
    ref = oracle_layout(orc, w)
    assert int(buf.status.cpu().numpy().view(np.uint32)[0]) == ref.status
    assert np.array_equal(buf.pair_slot.cpu().numpy()[:w.N], ref.pair_slot)
    assert np.array_equal(buf.row_src.cpu().numpy()[:buf.rows], ref.row_src)
    assert np.array_equal(buf.expert_offsets.cpu().numpy(), ref.expert_offsets)
    assert int(ws.count_nonzero()) == 0


def test_deterministic_repeat(orc):
    w = make_workload("mid_zipf")
    a = GpuRun(w)
    b = GpuRun(w)
    for key in ("pair_slot", "row_src", "out", "q8", "s8", "q4", "s4", "y"):
        assert np.array_equal(getattr(a, key), getattr(b, key)), key


# ------------------------------------------------------------ host checks
def test_host_argument_errors():
    prob = B.Problem(num_tokens=16, hidden=100, num_experts=8, top_k=2, num_segments=2,
                     recv_capacity=32)
    x = torch.zeros((16, 100), dtype=torch.bfloat16, device="cuda")
    out = torch.zeros((32, 100), dtype=torch.bfloat16, device="cuda")
    rs = torch.zeros(32, dtype=torch.int32, device="cuda")
    ps = torch.zeros((16, 2), dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_permute(prob, x, rs, ps, out)          # H % 8 != 0
    assert e.value.code == B.MOE_ERR_UNSUPPORTED_SHAPE
    prob.hidden = 96
    x2 = torch.zeros(16 * 96 + 8, dtype=torch.bfloat16, device="cuda")[1:].view(-1)[:16 * 96]
    with pytest.raises(B.MoeError) as e:
        B.moe_permute(prob, x2, rs, ps, out)         # misaligned hidden
    assert e.value.code == B.MOE_ERR_INVALID_ARG
    prob.num_segments = 3                            # E % S != 0
    buf_ws = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_dispatch_layout(prob, ps, rs, rs, rs, rs, ps, None, rs, buf_ws)
    assert e.value.code == B.MOE_ERR_UNSUPPORTED_SHAPE


@pytest.mark.parametrize("path", ["lookback", "two_pass"])
@pytest.mark.parametrize("cfg", ["tiny", "mid_zipf", "decode_capacity"])
def test_other_layout_paths_match_oracle(orc, cfg, path):
    w = make_workload(cfg)
    run = GpuRun(w, flags=LAYOUT_PATHS[path], quant=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)


@pytest.mark.parametrize("path", sorted(LAYOUT_PATHS))
@pytest.mark.parametrize("N,k,E", [(12500, 8, 64), (16384, 8, 256), (8191, 8, 256),
                                   (8193, 8, 256), (4097, 1, 3), (1025, 1, 7), (256, 8, 40),
                                   (2049, 1, 9)])
def test_layout_cluster_sizes(orc, N, k, E, path):
    """Pair counts around the size limits of the layout kernels: 1025 and
    2048 pairs (one CTA, 4 pairs per lane), 2049 and 4097 pairs (a cluster
    of 1-pair lanes), 65528 and 65544 pairs (one tile below and above
    sixteen tiles of 4096), 100000 and 131072 pairs (tiles of 8192 pairs),
    with a ragged last tile and masked, out-of-range and duplicate ids."""
    w = custom(N=N, H=32, E=E, k=k, S=1, seed=N + E, p_mask=0.05, p_bad=0.01,
               distinct=(N % 2 == 0), with_out=False)
    flags = B.MOE_FLAG_CHECK_DUPLICATES | LAYOUT_PATHS[path]
    run = GpuRun(w, flags=flags, quant=False, combine=False)
    ref = oracle_layout(orc, w, flags=orc.FLAG_CHECK_DUPLICATES)
    assert_layout(run, ref)


def test_cuda_graph_capture_and_replay(orc):
    """The whole path (layout, three permutes, combine) is captured once in a
    CUDA graph and replayed on new inputs written into the same buffers."""
    w1 = make_workload("mid_zipf", n_tokens=1536)
    w2 = make_workload("mid_zipf", n_tokens=1536, seed=77)
    prob = problem_of(w1)
    buf = poison_buffers(B.Buffers(prob))
    ids = torch.from_numpy(w1.ids).cuda()
    hidden = to_dev_bf16(w1.hidden)
    X = to_dev_bf16(w1.expert_out)
    gates = torch.from_numpy(w1.gates).cuda()
    gs = torch.tensor([w1.global_scale], dtype=torch.float32, device="cuda")
    y = poisoned_empty((w1.N, w1.H), torch.bfloat16)

    def path():
        B.layout(prob, ids, buf)
        B.moe_permute(prob, hidden, buf.row_src, buf.pair_slot, buf.out)
        B.moe_permute_quant_fp8(prob, hidden, buf.row_src, buf.pair_slot, buf.out_fp8,
                                buf.scales_fp8)
        B.moe_permute_quant_nvfp4(prob, hidden, buf.row_src, buf.pair_slot, gs, buf.out_fp4,
                                  buf.scales_fp4)
        B.moe_combine(prob, X, gates, buf.pair_slot, y)

    path()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        path()
    for w in (w2, w1, w2):
        ids.copy_(torch.from_numpy(w.ids))
        hidden.copy_(to_dev_bf16(w.hidden))
        X.copy_(to_dev_bf16(w.expert_out))
        gates.copy_(torch.from_numpy(w.gates))
        gs.fill_(w.global_scale)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_layout(orc, w)
        assert int(buf.status.item()) == 0
        assert np.array_equal(buf.pair_slot.cpu().numpy(), ref.pair_slot)
        assert np.array_equal(bf16_np(buf.out), orc.permute_bf16(w.hidden, ref.row_src))
        q, sc = orc.permute_fp8(w.hidden, ref.row_src)
        assert np.array_equal(buf.out_fp8.cpu().numpy(), q)
        q, sc = orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale)
        assert np.array_equal(buf.scales_fp4.cpu().numpy(), sc)
        assert np.array_equal(bf16_np(y), orc.combine(w.expert_out, w.gates, ref.pair_slot))


# ------------------------------------------------------------ rounding edges
def _bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _one_token_per_row(orc, rows_f32, gs=1.0):
    """Each row of rows_f32 is one token routed to one expert (k = 1), so the
    dispatch output is the rows in order; returns (workload, run, layout)."""
    N, H = rows_f32.shape
    ids = np.zeros((N, 1), np.int32)
    w = Workload(name="edge", N=N, H=H, E=1, k=1, S=1, recv_capacity=N, expert_capacity=0,
                 ids=ids, gates=np.ones((N, 1), np.float32), hidden=_bits(rows_f32),
                 expert_out=None, global_scale=float(np.float32(gs)), seed=0)
    run = GpuRun(w, combine=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    return w, run, ref


def test_fp8_rounding_ties_and_edges(orc):
    """Quotients exactly on E4M3 midpoints (ties to even), on codes, in the
    subnormal range, at the saturation edge and signed zeros: the block scale
    is a power of two, so x / scale is exact."""
    mids = np.array([8.5, 9.5, 17, 19, 36, 40, 104, 232, 240, 1.0625, 1.1875,
                     0.0029296875, 0.0048828125, 0.0068359375, 0.0009765625], np.float32)
    codes = np.array([16, 18, 448, 0.015625, 0.001953125, 2.0, 3.5], np.float32)
    rng = np.random.default_rng(3)
    rows = []
    for k in range(-6, 6):
        for sign in (1, -1):
            blk = np.zeros(128, np.float32)
            blk[0] = 448.0                                   # amax -> scale 2^k
            vals = np.concatenate([mids, -mids, codes, [-0.0, 0.0]])
            blk[1:1 + vals.size] = vals
            blk[1 + vals.size:] = rng.standard_normal(127 - vals.size) * 50
            rows.append(sign * blk * np.float32(2.0 ** k))
    x = np.stack(rows).reshape(-1, 256)
    w, run, ref = _one_token_per_row(orc, x)
    q, s = orc.permute_fp8(w.hidden, ref.row_src)
    assert np.array_equal(run.q8, q)
    assert np.array_equal(run.s8.view(np.uint32), s.view(np.uint32))


@pytest.mark.parametrize("gs", [1.0, 1.0 + 2.0 ** -23, 1.0 - 2.0 ** -24, 1.0 + 2.0 ** -22,
                                0.3333333432674408, 2.0 ** -7])
def test_nvfp4_rounding_ties_and_near_ties(orc, gs):
    """Blocks whose amax makes the decode scale d = float(e4m3 scale) * gs
    equal to gs (amax = 6 * gs-ish), with elements on E2M1 midpoints: with gs
    a power of two the quotients are exact ties; with gs one ulp off 1 they
    are one or two ulps off the midpoints, where a reciprocal product and the
    division can round differently."""
    mids = np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0, 0.5, 1.0, 1.5, 2, 3, 4, 6,
                     0.125], np.float32)
    rows = []
    rng = np.random.default_rng(int(gs * 1000) % 97)
    scale_of = np.float32(6.0) * np.float32(gs) if gs < 0.9 else np.float32(6.0)
    for sign in (1, -1):
        for r in range(8):
            blk = np.zeros(32, np.float32)
            blk[0] = scale_of
            blk[1:1 + mids.size] = mids * (np.float32(gs) if gs < 0.9 else 1)
            blk[16] = scale_of
            blk[17:] = rng.uniform(-6, 6, 15) * (np.float32(gs) if gs < 0.9 else 1)
            rows.append(sign * blk)
    x = np.stack(rows)
    w, run, ref = _one_token_per_row(orc, x, gs=gs)
    q, s = orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale)
    assert np.array_equal(run.s4, s)
    assert np.array_equal(run.q4, q)


# ------------------------------------------------------------ expert padding
PAD_EDGE = {
    "pad4_masked": (dict(N=1000, H=256, E=16, k=4, S=4, C=1000 * 4 + 16 * 3, p_mask=0.1), 4),
    "pad128": (dict(N=2048, H=512, E=64, k=8, S=8, C=2048 * 8 + 64 * 127), 128),
    "pad16_overflow": (dict(N=500, H=128, E=8, k=2, S=2, C=900), 16),
    "pad3_badids": (dict(N=3001, H=96, E=40, k=3, S=5, C=3001 * 3 + 80, p_bad=0.02), 3),
}


@pytest.mark.parametrize("path", sorted(LAYOUT_PATHS))
@pytest.mark.parametrize("name", sorted(PAD_EDGE))
def test_expert_padding_parity(orc, name, path):
    spec, pad = PAD_EDGE[name]
    w = custom(seed=zlib.crc32(name.encode()) % 1000, **spec)
    flags = B.MOE_FLAG_CHECK_DUPLICATES | LAYOUT_PATHS[path]
    run = GpuRun(w, flags=flags, pad=pad)
    ref = oracle_layout(orc, w, flags=orc.FLAG_CHECK_DUPLICATES, pad=pad)
    assert_layout(run, ref)
    assert np.all(ref.expert_offsets % pad == 0)
    assert_all_outputs(orc, w, run, ref)


# ------------------------------------------------------------ random sweep
def _random_spec(i):
    """A seeded random problem: any mode (packed, padded, capacity), masked
    and out-of-range ids, duplicates, ragged sizes."""
    rng = np.random.default_rng(7000 + i)
    E = int(rng.choice([1, 3, 8, 24, 64, 160, 256]))
    divisors = [d for d in range(1, E + 1) if E % d == 0]
    S = int(rng.choice(divisors))
    k = int(rng.integers(1, min(16, E) + 1)) if rng.random() < 0.8 else int(rng.integers(1, 17))
    N = int(rng.choice([0, 1, 2, 31, 257, 1000, 3333]))
    H = int(32 * rng.choice([1, 3, 4, 7, 12, 16]))
    spec = dict(N=N, H=H, E=E, k=k, S=S, p_mask=float(rng.choice([0, 0.05, 0.5])),
                p_bad=float(rng.choice([0, 0, 0.02])), distinct=k <= E and rng.random() < 0.8)
    mode = rng.choice(["packed", "padded", "capacity"])
    pad = 0
    if mode == "capacity":
        spec["Ce"] = int(rng.integers(1, max(2, 2 * N * k // max(E, 1) + 2)))
    elif mode == "padded":
        pad = int(rng.choice([2, 4, 8, 128]))
        spec["C"] = N * k + E * (pad - 1) - int(rng.integers(0, 3))
    else:
        spec["C"] = max(0, int(N * k * rng.uniform(0.8, 1.2)))
    return spec, pad, bool(rng.random() < 0.5), bool(rng.random() < 0.4)


def _check_peer_sends(orc, w, run, ref, rng):
    """The bf16, FP8 (H % 128 == 0) and NVFP4 dispatches sent to S stand-in
    receive buffers at random put offsets: each segment of the oracle's
    dispatch output lands at its offset bit for bit, every other row of every
    buffer keeps its poison; the combine reading the bf16 rows back from the
    buffers equals the oracle's combine of the dispatch output."""
    from gpu_util import BF16_POISON, BYTE_POISON, F32_POISON
    H, S = w.H, w.S
    L = w.E // S
    if w.expert_capacity > 0:
        starts = [s * L * w.expert_capacity for s in range(S)]
        seg_rows = [L * w.expert_capacity] * S
    else:
        starts = [int(v) // H for v in ref.meta[1]]
        seg_rows = [int(v) // H for v in ref.meta[0]]
    put = [int(v) for v in rng.integers(0, 40, S)]
    hid = to_dev_bf16(w.hidden) if w.N > 0 else torch.empty((1, H), dtype=torch.bfloat16,
                                                             device="cuda")
    put_d = torch.tensor(put, dtype=torch.int64, device="cuda")
    gs = torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")

    def bufs(width, dtype):
        return [poisoned_empty((put[s] + seg_rows[s] + 3, width), dtype) for s in range(S)]

    def ptrs(ts):
        return torch.tensor([t.data_ptr() for t in ts], dtype=torch.int64, device="cuda")

    cases = [("bf16", (H, torch.bfloat16), None)]
    if H % 128 == 0:
        cases.append(("fp8", (H, torch.uint8), (H // 128, torch.float32)))
    cases.append(("nvfp4", (H // 2, torch.uint8), (H // 16, torch.uint8)))
    for fmt, code_spec, scale_spec in cases:
        codes = bufs(*code_spec)
        scales = bufs(*scale_spec) if scale_spec else None
        if fmt == "bf16":
            B.moe_permute_to_peers(run.prob, hid, run.buf.row_src, run.buf.pair_slot,
                                   run.buf.meta, ptrs(codes), put_d)
            want = [orc.permute_bf16(w.hidden, ref.row_src)]
            if w.N > 0:
                # and back: the combine reading the rows where they landed
                y = poisoned_empty((w.N, H), torch.bfloat16)
                B.moe_combine_from_peers(run.prob, ptrs(codes), put_d, run.buf.meta,
                                         torch.from_numpy(w.gates).cuda(), run.buf.pair_slot, y)
                torch.cuda.synchronize()
                assert np.array_equal(bf16_np(y), orc.combine(want[0], w.gates, ref.pair_slot))
        elif fmt == "fp8":
            B.moe_permute_quant_fp8_to_peers(run.prob, hid, run.buf.row_src, run.buf.pair_slot,
                                             run.buf.meta, ptrs(codes), ptrs(scales), put_d)
            q, sc = orc.permute_fp8(w.hidden, ref.row_src)
            want = [q, sc.view(np.uint32)]
        else:
            B.moe_permute_quant_nvfp4_to_peers(run.prob, hid, run.buf.row_src,
                                               run.buf.pair_slot, run.buf.meta, gs,
                                               ptrs(codes), ptrs(scales), put_d)
            want = list(orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale))
        torch.cuda.synchronize()
        R = ref.row_src.size
        for s in range(S):
            # a padded layout whose recv_capacity cuts the last expert block
            # short has segment rows past the last local row: those are not
            # written (moe_dc.h), and keep their poison
            n = max(0, min(starts[s] + seg_rows[s], R) - starts[s])
            lo, hi = put[s], put[s] + n
            got = [codes[s].view(torch.int16).cpu().numpy().view(np.uint16) if fmt == "bf16"
                   else codes[s].cpu().numpy()]
            poison_of = [BF16_POISON if fmt == "bf16" else BYTE_POISON]
            if scales is not None:
                sv = scales[s].cpu().numpy()
                got.append(sv.view(np.uint32) if fmt == "fp8" else sv)
                poison_of.append(np.uint32(F32_POISON) if fmt == "fp8" else BYTE_POISON)
            for g, wnt, p in zip(got, want, poison_of):
                assert np.array_equal(g[lo:hi], wnt[starts[s]:starts[s] + n]), (fmt, s)
                assert np.all(g[:lo] == p) and np.all(g[hi:] == p), (fmt, s)


@pytest.mark.parametrize("i", range(40))
def test_random_problem_sweep(orc, i):
    spec, pad, two_pass, swizzled = _random_spec(i)
    w = custom(seed=100 + i, **spec)
    path = "two_pass" if two_pass else ("lookback", "auto")[i % 2]
    flags = B.MOE_FLAG_CHECK_DUPLICATES | LAYOUT_PATHS[path] | \
        (B.MOE_FLAG_NVFP4_SWIZZLED_SCALES if swizzled else 0)
    run = GpuRun(w, flags=flags, pad=pad)
    ref = oracle_layout(orc, w, flags=orc.FLAG_CHECK_DUPLICATES, pad=pad)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)
    rows = run.buf.rows
    if rows == 0:
        return
    rng = np.random.default_rng(9000 + i)
    # SwiGLU of the dispatch rows: random width, format and gate/up layout
    I = 32 * int(rng.integers(1, 24))
    fmt, inter = int(rng.integers(0, 6)), bool(rng.random() < 0.5)
    gu = _bits(rng.standard_normal((rows, 2 * I)) * 2)
    codes, scales = (poison(t) for t in B.swiglu_buffers(rows, I, fmt))
    gs = torch.tensor([0.02], dtype=torch.float32, device="cuda")
    B.moe_swiglu_quant(run.prob, I, fmt, int(inter), to_dev_bf16(gu), run.buf.row_src, gs,
                       codes, scales)
    # dispatch backward of a random row gradient
    g_rows = _bits(rng.standard_normal((rows, w.H)))
    gh = poisoned_empty((max(w.N, 1), w.H), torch.bfloat16)
    if w.N > 0:
        B.moe_permute_backward(run.prob, to_dev_bf16(g_rows), run.buf.pair_slot, gh)
    torch.cuda.synchronize()
    want_c, want_s = orc.swiglu_quant(gu, ref.row_src, fmt, interleaved=inter, global_scale=0.02)
    assert np.array_equal(codes.cpu().numpy(), want_c), (fmt, inter)
    if fmt != B.MOE_QUANT_BF16:
        assert np.array_equal(scales.cpu().numpy(), want_s), (fmt, inter)
    if w.N > 0:
        assert np.array_equal(bf16_np(gh), orc.permute_backward(g_rows, ref.pair_slot))
    # the sends to peers (not in overflow: a segment would then run past rows)
    if not (ref.status & orc.STATUS_CAPACITY) and not swizzled:
        _check_peer_sends(orc, w, run, ref, rng)


# ------------------------------------------------------------ scale atom layout
@pytest.mark.parametrize("spec", [
    dict(N=700, H=96, E=8, k=3, S=2, p_mask=0.2),          # 6 scale columns: column padding
    dict(N=300, H=256, E=4, k=2, S=1, C=1000, p_mask=0.1),  # rows not a multiple of 128
    dict(N=64, H=7168, E=256, k=8, S=8),
], ids=["H96", "rows1000", "H7168"])
def test_nvfp4_swizzled_scales(orc, spec):
    w = custom(seed=5, **spec)
    run = GpuRun(w, flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES, combine=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    q, s_lin = orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale)
    assert np.array_equal(run.q4, q)
    assert np.array_equal(run.s4, orc.swizzle_scales(s_lin))
    q, s_lin = orc.permute_mxfp4(w.hidden, ref.row_src)
    assert np.array_equal(run.qmx, q)
    assert np.array_equal(run.smx, orc.swizzle_scales(s_lin))


def test_nvfp4_swizzled_scales_workload(orc):
    w = make_workload("mid_zipf")
    run = GpuRun(w, flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES, combine=False)
    ref = oracle_layout(orc, w)
    q, s_lin = orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale)
    assert np.array_equal(run.q4, q)
    assert np.array_equal(run.s4, orc.swizzle_scales(s_lin))


# ------------------------------------------------------------ backward
@pytest.mark.parametrize("cfg,n", [("tiny", None), ("mid_zipf", 1024), ("decode_capacity", None),
                                   ("fp8_metric", 1024)])
def test_backward_parity(orc, cfg, n):
    w = make_workload(cfg, n_tokens=n)
    run = GpuRun(w, quant=False, combine=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    prob = run.prob
    rows = run.buf.rows
    rng = np.random.default_rng(23)
    g_rows = _bits(rng.standard_normal((rows, w.H)))
    g_tok = _bits(rng.standard_normal((w.N, w.H)))
    # dispatch backward: bit-exact (fp32 adds in j order, one bf16 rounding)
    gh = poisoned_empty((w.N, w.H), torch.bfloat16)
    B.moe_permute_backward(prob, to_dev_bf16(g_rows), run.buf.pair_slot, gh)
    # combine backward: bit-exact expert-row gradients, gate gradients within
    # the fp32 accumulation bound of the exact dot products
    gx = poisoned_empty((rows, w.H), torch.bfloat16)
    gw = poisoned_empty((w.N, w.k), torch.float32)
    X = w.expert_out
    B.moe_combine_backward(prob, to_dev_bf16(g_tok), to_dev_bf16(X),
                           torch.from_numpy(w.gates).cuda(), run.buf.pair_slot, run.buf.row_src,
                           gx, gw)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_np(gh), orc.permute_backward(g_rows, ref.pair_slot))
    ogx, ogw = orc.combine_backward(g_tok, X, w.gates, ref.pair_slot)
    assert np.array_equal(bf16_np(gx), ogx)
    gw_gpu = gw.cpu().numpy()
    f = lambda b: (b.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    mag = np.zeros_like(ogw, dtype=np.float64)
    for j in range(w.k):
        s = ref.pair_slot[:, j]
        ok = s >= 0
        mag[:, j] = np.where(ok, np.sum(np.abs(f(g_tok) * f(X[np.maximum(s, 0)])), axis=1), 0)
    bound = 2.0 ** -24 * (w.H / 32 + 8) * mag + 2.0 ** -23 * np.abs(ogw)
    assert np.all(np.abs(gw_gpu.astype(np.float64) - ogw) <= bound)
    assert np.all(gw_gpu[ref.pair_slot < 0] == 0)


# ------------------------------------------------------------ SwiGLU + requant
@pytest.mark.parametrize("fmt", [0, 1, 2, 3, 4, 5],
                         ids=["nvfp4", "mxfp8", "mxfp4", "bf16", "mxfp6e2m3", "mxfp6e3m2"])
@pytest.mark.parametrize("interleaved", [False, True], ids=["split", "interleaved"])
@pytest.mark.parametrize("I", [2048, 96 * 32 + 32])
def test_swiglu_quant_parity(orc, fmt, interleaved, I):
    w = make_workload("mid_zipf", n_tokens=256, with_expert_out=False)
    C = w.N * w.k + 100                       # some rows without a token
    w = Workload(**{**w.__dict__, "recv_capacity": C})
    run = GpuRun(w, quant=False, combine=False)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    rng = np.random.default_rng(31 + I + fmt)
    gu = _bits(rng.standard_normal((C, 2 * I)) * np.float32(2.5))
    gu[3, :8] = _bits(np.array([0, -0.0, 30, -30, 90, -90, 1e-3, -1e-3], np.float32))
    gu[5, :I] = 0x8000                        # gate -0: a row of -0 outputs (all-zero blocks)
    gu[5, I:] = 0x3F80
    gu[6, :64] = 0                            # two zero blocks at the start of a row
    codes, scales = (poison(t) for t in B.swiglu_buffers(C, I, fmt))
    gs = torch.tensor([0.01], dtype=torch.float32, device="cuda")
    B.moe_swiglu_quant(run.prob, I, fmt, int(interleaved), to_dev_bf16(gu), run.buf.row_src,
                       gs, codes, scales)
    torch.cuda.synchronize()
    want_c, want_s = orc.swiglu_quant(gu, ref.row_src, fmt, interleaved=interleaved,
                                      global_scale=0.01)
    assert np.array_equal(codes.cpu().numpy(), want_c)
    if fmt != B.MOE_QUANT_BF16:                # bf16 output has no scales
        assert np.array_equal(scales.cpu().numpy(), want_s)


def test_swiglu_exp_matches_oracle_bitwise(orc):
    """The kernel's e^x sequence is the oracle's: silu(g) * 1 over a dense
    sweep of bf16 gate values, MXFP8-coded with a power-of-two block scale,
    so any difference in e^x at the codes' resolution shows."""
    I = 1024
    g = np.arange(-(1 << 15), 1 << 15, dtype=np.int64).astype(np.uint16)  # every bf16 pattern
    g = g[((g >> 7) & 0xFF) != 0xFF]                                    # drop inf / NaN
    rows = len(g) // I
    g = g[:rows * I].reshape(rows, I)
    u = np.full((rows, I), 0x3F80, np.uint16)                           # 1.0
    gu = np.ascontiguousarray(np.concatenate([g, u], axis=1))
    ids = np.zeros((rows, 1), np.int32)
    ww = Workload(name="sweep", N=rows, H=64, E=1, k=1, S=1, recv_capacity=rows,
                  expert_capacity=0, ids=ids, gates=np.ones((rows, 1), np.float32),
                  hidden=np.zeros((rows, 64), np.uint16), expert_out=None, global_scale=1.0,
                  seed=0)
    run = GpuRun(ww, quant=False, combine=False)
    for fmt in (0, 1):
        codes, scales = (poison(t) for t in B.swiglu_buffers(rows, I, fmt))
        gs = torch.tensor([1.0], dtype=torch.float32, device="cuda")
        B.moe_swiglu_quant(run.prob, I, fmt, 0, to_dev_bf16(gu), run.buf.row_src, gs, codes,
                           scales)
        torch.cuda.synchronize()
        want_c, want_s = orc.swiglu_quant(gu, np.arange(rows, dtype=np.int32), fmt,
                                          global_scale=1.0)
        assert np.array_equal(codes.cpu().numpy(), want_c)
        assert np.array_equal(scales.cpu().numpy(), want_s)


@pytest.mark.parametrize("gscale", [1e-33, 2e-6, 0.37, 3e4, 1e36])
def test_swiglu_quant_wide_range(orc, gscale):
    """Gate/up values drawn from every finite bf16 bit pattern (all binades,
    subnormals, signed zeros) and global scales from tiny to huge: NVFP4
    blocks then take every path of the quotient (the corrected reciprocal,
    the division fallback for a tiny or huge block scale, the clamp of
    quotients above 8), and MX blocks every E8M0 clamp."""
    I = 1024
    rows = 96
    rng = np.random.default_rng(int(gscale * 1e3) % 1000 + 7)
    gu = rng.integers(0, 1 << 16, size=(rows, 2 * I), dtype=np.uint32).astype(np.uint16)
    # exponent fields above 189 (|x| >= 2^63, inf, NaN) folded down, so that
    # gate * up stays finite
    ex = (gu >> 7) & 0xFF
    gu = (gu & 0x807F) | (np.where(ex > 189, ex - 66, ex) << 7).astype(np.uint16)
    # some rows of one narrow binade so that a block's amax sits near its values
    gu[::7, :] = (gu[::7, :] & 0x807F) | 0x3F00
    # a row near the top of the fp32 range: block scales above 2^124
    gu[5, :] = 0x5F7F
    ids = np.zeros((rows, 1), np.int32)
    ww = Workload(name="wide", N=rows, H=64, E=1, k=1, S=1, recv_capacity=rows,
                  expert_capacity=0, ids=ids, gates=np.ones((rows, 1), np.float32),
                  hidden=np.zeros((rows, 64), np.uint16), expert_out=None, global_scale=1.0,
                  seed=0)
    run = GpuRun(ww, quant=False, combine=False)
    for fmt in (0, 1, 2, 3, 4, 5):
        for layout in (0, 1):                      # split, interleaved
            codes, scales = (poison(t) for t in B.swiglu_buffers(rows, I, fmt))
            gs = torch.tensor([gscale], dtype=torch.float32, device="cuda")
            B.moe_swiglu_quant(run.prob, I, fmt, layout, to_dev_bf16(gu), run.buf.row_src, gs,
                               codes, scales)
            torch.cuda.synchronize()
            want_c, want_s = orc.swiglu_quant(gu, np.arange(rows, dtype=np.int32), fmt,
                                              interleaved=bool(layout),
                                              global_scale=float(np.float32(gscale)))
            if fmt != B.MOE_QUANT_BF16:
                assert np.array_equal(scales.cpu().numpy(), want_s), (fmt, layout)
            assert np.array_equal(codes.cpu().numpy(), want_c), (fmt, layout)


# ------------------------------------------------------------ concurrency
def test_concurrent_streams_from_two_threads(orc):
    """Two host threads, each on its own CUDA stream with its own buffers and
    workspace, run the whole step (layout, three permutes, combine) on
    different problems at the same time, five times each: every output of
    the last pass matches the oracle.  The library keeps no device state
    between calls, and its host-side caches are shared safely."""
    import threading
    ws = [make_workload("mid_zipf", n_tokens=1024),
          custom(N=777, H=256, E=24, k=3, S=4, seed=77, p_mask=0.05, p_bad=0.01)]
    runs = [None, None]
    errors = []

    def work(i):
        try:
            stream = torch.cuda.Stream()
            with torch.cuda.stream(stream):
                for _ in range(5):
                    runs[i] = GpuRun(ws[i])
        except Exception as e:  # reported below, on the main thread
            errors.append(e)

    threads = [threading.Thread(target=work, args=(i,)) for i in range(2)]
    for t in threads:
        t.start()
    for t in threads:
        t.join()
    assert not errors, errors
    for w, run in zip(ws, runs):
        ref = oracle_layout(orc, w)
        assert_layout(run, ref)
        assert_all_outputs(orc, w, run, ref)


# ------------------------------------------------------------ dispatch to peers
@pytest.mark.parametrize("mode", ["packed", "padded", "capacity"])
def test_permute_to_peers(orc, mode):
    """moe_permute_to_peers with S local buffers standing in for the S
    ranks' receive buffers: segment s of the oracle's dispatch output lands
    at rows [put[s], put[s] + rows_s) of buffer s, bit for bit (padding rows
    inside a segment as zeros), and every other row of every buffer keeps
    its poison (no stray store)."""
    spec = dict(N=1500, H=264, E=24, k=3, S=4, p_mask=0.05, p_bad=0.01)
    pad = 0
    if mode == "padded":
        pad = 8
        spec["C"] = 1500 * 3 + 24 * 7
    elif mode == "capacity":
        spec["Ce"] = 150
    w = custom(seed=31, with_out=False, **spec)
    run = GpuRun(w, quant=False, combine=False, pad=pad)
    ref = oracle_layout(orc, w, pad=pad)
    assert_layout(run, ref)
    want = orc.permute_bf16(w.hidden, ref.row_src)
    L = w.E // w.S
    if mode == "capacity":
        starts = [s * L * w.expert_capacity for s in range(w.S)]
        seg_rows = [L * w.expert_capacity] * w.S
    else:
        starts = [int(v) // w.H for v in ref.meta[1]]
        seg_rows = [int(v) // w.H for v in ref.meta[0]]
    rng = np.random.default_rng(9)
    put = [int(rng.integers(0, 300)) for _ in range(w.S)]
    bufs = [poisoned_empty((put[s] + seg_rows[s] + 17, w.H), torch.bfloat16)
            for s in range(w.S)]
    peer = torch.tensor([b.data_ptr() for b in bufs], dtype=torch.int64, device="cuda")
    put_d = torch.tensor(put, dtype=torch.int64, device="cuda")
    B.moe_permute_to_peers(run.prob, to_dev_bf16(w.hidden), run.buf.row_src, run.buf.pair_slot,
                           run.buf.meta, peer, put_d)
    torch.cuda.synchronize()
    from gpu_util import BF16_POISON
    for s in range(w.S):
        got = bf16_np(bufs[s])
        seg = want[starts[s]:starts[s] + seg_rows[s]]
        assert np.array_equal(got[put[s]:put[s] + seg_rows[s]], seg), s
        untouched = np.concatenate([got[:put[s]], got[put[s] + seg_rows[s]:]])
        assert np.all(untouched == BF16_POISON), s


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("mode", ["packed", "padded", "capacity"])
def test_quantised_permute_to_peers(orc, mode, fmt):
    """moe_permute_quant_fp8_to_peers / moe_permute_quant_nvfp4_to_peers with
    S local code and scale buffers standing in for the S ranks' receive
    buffers: segment s of the oracle's FP8 / NVFP4 dispatch (codes and
    row-major scales) lands at rows [put[s], put[s] + rows_s) of rank s's
    buffers, bit for bit (padding rows inside a segment as zeros), and every
    other row of every buffer keeps its poison."""
    spec = dict(N=1500, H=384, E=24, k=3, S=4, p_mask=0.05, p_bad=0.01)
    pad = 0
    if mode == "padded":
        pad = 8
        spec["C"] = 1500 * 3 + 24 * 7
    elif mode == "capacity":
        spec["Ce"] = 150
    w = custom(seed=41, with_out=False, **spec)
    run = GpuRun(w, quant=False, combine=False, pad=pad)
    ref = oracle_layout(orc, w, pad=pad)
    assert_layout(run, ref)
    H = w.H
    if fmt == "fp8":
        q_want, s_want = orc.permute_fp8(w.hidden, ref.row_src)
        s_want = s_want.view(np.uint32)
        code_w, scale_w, scale_dt = H, H // 128, torch.float32
    else:
        q_want, s_want = orc.permute_nvfp4(w.hidden, ref.row_src, w.global_scale)
        code_w, scale_w, scale_dt = H // 2, H // 16, torch.uint8
    L = w.E // w.S
    if mode == "capacity":
        starts = [s * L * w.expert_capacity for s in range(w.S)]
        seg_rows = [L * w.expert_capacity] * w.S
    else:
        starts = [int(v) // H for v in ref.meta[1]]
        seg_rows = [int(v) // H for v in ref.meta[0]]
    rng = np.random.default_rng(13)
    put = [int(rng.integers(0, 300)) for _ in range(w.S)]
    codes = [poisoned_empty((put[s] + seg_rows[s] + 17, code_w), torch.uint8)
             for s in range(w.S)]
    scales = [poisoned_empty((put[s] + seg_rows[s] + 17, scale_w), scale_dt)
              for s in range(w.S)]
    pc = torch.tensor([t.data_ptr() for t in codes], dtype=torch.int64, device="cuda")
    psc = torch.tensor([t.data_ptr() for t in scales], dtype=torch.int64, device="cuda")
    put_d = torch.tensor(put, dtype=torch.int64, device="cuda")
    hid = to_dev_bf16(w.hidden)
    if fmt == "fp8":
        B.moe_permute_quant_fp8_to_peers(run.prob, hid, run.buf.row_src, run.buf.pair_slot,
                                         run.buf.meta, pc, psc, put_d)
    else:
        gs = torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")
        B.moe_permute_quant_nvfp4_to_peers(run.prob, hid, run.buf.row_src, run.buf.pair_slot,
                                           run.buf.meta, gs, pc, psc, put_d)
    torch.cuda.synchronize()
    from gpu_util import BYTE_POISON, F32_POISON
    for s in range(w.S):
        lo, hi = put[s], put[s] + seg_rows[s]
        got_q = codes[s].cpu().numpy()
        got_s = scales[s].cpu().numpy()
        if fmt == "fp8":
            got_s = got_s.view(np.uint32)
            s_poison = np.uint32(F32_POISON)
        else:
            s_poison = BYTE_POISON
        assert np.array_equal(got_q[lo:hi], q_want[starts[s]:starts[s] + seg_rows[s]]), s
        assert np.array_equal(got_s[lo:hi], s_want[starts[s]:starts[s] + seg_rows[s]]), s
        assert np.all(np.concatenate([got_q[:lo], got_q[hi:]]) == BYTE_POISON), s
        assert np.all(np.concatenate([got_s[:lo], got_s[hi:]]) == s_poison), s


@pytest.mark.parametrize("mode", ["packed", "padded", "capacity"])
def test_combine_from_peers(orc, mode):
    """moe_combine_from_peers with S local buffers standing in for the S
    ranks' expert-output buffers: segment s of the expert outputs sits at
    rows [get[s], get[s] + rows_s) of buffer s (poison elsewhere); the result
    equals the oracle's combine of the local expert outputs, bit for bit."""
    spec = dict(N=1500, H=264, E=24, k=3, S=4, p_mask=0.05, p_bad=0.01)
    pad = 0
    if mode == "padded":
        pad = 8
        spec["C"] = 1500 * 3 + 24 * 7
    elif mode == "capacity":
        spec["Ce"] = 150
    w = custom(seed=47, **spec)
    run = GpuRun(w, quant=False, combine=False, pad=pad)
    ref = oracle_layout(orc, w, pad=pad)
    assert_layout(run, ref)
    L = w.E // w.S
    if mode == "capacity":
        starts = [s * L * w.expert_capacity for s in range(w.S)]
        seg_rows = [L * w.expert_capacity] * w.S
    else:
        starts = [int(v) // w.H for v in ref.meta[1]]
        seg_rows = [int(v) // w.H for v in ref.meta[0]]
    rng = np.random.default_rng(21)
    get = [int(rng.integers(0, 300)) for _ in range(w.S)]
    X = w.expert_out
    bufs = []
    for s in range(w.S):
        b = np.full((get[s] + seg_rows[s] + 9, w.H), 0x7FC1, np.uint16)
        b[get[s]:get[s] + seg_rows[s]] = X[starts[s]:starts[s] + seg_rows[s]]
        bufs.append(to_dev_bf16(b))
    peer = torch.tensor([t.data_ptr() for t in bufs], dtype=torch.int64, device="cuda")
    get_d = torch.tensor(get, dtype=torch.int64, device="cuda")
    y = poisoned_empty((w.N, w.H), torch.bfloat16)
    B.moe_combine_from_peers(run.prob, peer, get_d, run.buf.meta,
                             torch.from_numpy(w.gates).cuda(), run.buf.pair_slot, y)
    torch.cuda.synchronize()
    assert np.array_equal(bf16_np(y), orc.combine(X, w.gates, ref.pair_slot))


def test_quantised_permute_to_peers_rejects_the_atom_layout():
    w = custom(N=64, H=256, E=8, k=2, S=2, seed=3, with_out=False)
    prob = problem_of(w, flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES)
    z = torch.zeros(1 << 16, dtype=torch.uint8, device="cuda")
    i32 = torch.zeros(1 << 12, dtype=torch.int32, device="cuda")
    p64 = torch.zeros(w.S, dtype=torch.int64, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_permute_quant_nvfp4_to_peers(prob, z, i32, i32, i32, i32.view(torch.float32),
                                           p64, p64, p64)
    assert e.value.code == B.MOE_ERR_UNSUPPORTED_SHAPE


def test_grouped_gemm_ready_dispatch_full_size(orc):
    """The f1 configuration the benchmark times: the metric workload with
    experts padded to 128 rows (recv_capacity = N*k + 127*E) and FP4 scales
    in the atom layout; every row, code and scale byte against the oracle."""
    w = make_workload("fp8_metric", with_expert_out=False)
    pad = 128
    w = Workload(**{**w.__dict__, "recv_capacity": w.N * w.k + w.E * (pad - 1)})
    run = GpuRun(w, flags=B.MOE_FLAG_NVFP4_SWIZZLED_SCALES, combine=False, pad=pad)
    ref = oracle_layout(orc, w, pad=pad)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)
