"""Cases for the build with per-CTA trace records (libmoedc_trace.so).

Not collected by default: tests/test_gpu_trace_build.py runs this file in a
child process whose MOE_LIB_PATH names that build.  The records of a whole
step and of each layout kernel, the counter running past the capacity,
detaching, argument errors, and the kernels of the NEXT-row calls."""
import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200 import trace as T
from combine_topk_ids_scan_b200.inputs import make_workload
from gpu_util import BYTE_POISON, GpuRun, poisoned_empty, to_dev_bf16
from test_gpu_parity import assert_all_outputs, assert_layout, oracle_layout
from trace_checks import check_launches

pytestmark = pytest.mark.gpu

LAYOUT_NAMES = {T.KERNELS[i] for i in T.LAYOUT_KERNELS}


@pytest.fixture(scope="module", autouse=True)
def _trace_build():
    assert torch.cuda.is_available(), "the trace cases need a CUDA device"
    assert "trace records" in B.version(), f"not the trace build: {B.version()}"


def test_a_traced_step_matches_the_oracle_and_records_every_cta(orc):
    w = make_workload("mid_zipf")
    with T.Tracer() as tr:
        run = GpuRun(w)
    ref = oracle_layout(orc, w)
    assert_layout(run, ref)
    assert_all_outputs(orc, w, run, ref)
    ls = check_launches(tr)
    names = [launch.kernel for launch in ls]
    assert names[0] in LAYOUT_NAMES
    assert names[1:] == ["permute_bf16", "permute_fp8", "permute_nvfp4", "permute_mxfp4",
                         "combine"]
    assert [launch.variant for launch in ls[3:5]] == [0, 0]     # linear scales
    assert ls[5].variant == 8                                     # combine KMAX for k = 6
    for launch in ls[1:]:
        assert launch.ctas > 1 and launch.sms > 1


@pytest.mark.parametrize("cfg,flags,want", [
    ("decode_capacity", 0, ["layout_single"]),
    ("mid_zipf", 0, ["layout_cluster"]),
    ("mid_zipf", B.MOE_FLAG_LAYOUT_LOOKBACK, ["layout_lookback"]),
    ("mid_zipf", B.MOE_FLAG_LAYOUT_TWO_PASS, ["layout_scan", "layout_emit"]),
])
def test_each_layout_kernel_records(orc, cfg, flags, want):
    w = make_workload(cfg)
    with T.Tracer() as tr:
        run = GpuRun(w, flags=flags, quant=False, combine=False)
    assert_layout(run, oracle_layout(orc, w))
    names = [launch.kernel for launch in check_launches(tr)]
    assert names == want + ["permute_bf16"]


def _permute_once(run, w, stream=None):
    B.moe_permute(run.prob, to_dev_bf16(w.hidden), run.buf.row_src, run.buf.pair_slot,
                  run.buf.out, stream)


def test_counter_runs_past_the_capacity_and_nothing_is_written_beyond_it():
    w = make_workload("mid_zipf", with_expert_out=False)
    run = GpuRun(w, quant=False, combine=False)
    with T.Tracer() as tr:
        _permute_once(run, w)
    (full,) = check_launches(tr)
    assert full.ctas > 4
    raw = torch.full((64 * 32,), BYTE_POISON, dtype=torch.uint8, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.moe_trace_attach(raw[:4 * 32], count)
    _permute_once(run, w)
    B.moe_trace_attach(None, None)
    torch.cuda.synchronize()
    n = int(count.item())
    assert n == full.ctas
    host = raw.cpu().numpy()
    assert np.all(host[4 * 32:] == BYTE_POISON)
    recs = T.decode(host[:4 * 32], n)
    assert recs.size == 4 and np.all(recs["kernel"] == 6)
    assert len(set(recs["block"].tolist())) == 4


def test_detach_stops_recording():
    w = make_workload("tiny", with_expert_out=False)
    run = GpuRun(w, quant=False, combine=False)
    raw = torch.zeros(1 << 15, dtype=torch.uint8, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    B.moe_trace_attach(raw, count)
    _permute_once(run, w)
    B.moe_trace_attach(None, None)
    torch.cuda.synchronize()
    once = int(count.item())
    assert once > 0
    _permute_once(run, w)
    torch.cuda.synchronize()
    assert int(count.item()) == once


def test_graph_replays_record():
    """Kernels captured into a CUDA graph record on every replay (the
    attachment is read by the kernels when they run)."""
    w = make_workload("tiny", with_expert_out=False)
    run = GpuRun(w, quant=False, combine=False)
    hidden = to_dev_bf16(w.hidden)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=side):
        B.moe_permute(run.prob, hidden, run.buf.row_src, run.buf.pair_slot, run.buf.out)
    with T.Tracer() as tr:
        _permute_once(run, w)
    (one,) = check_launches(tr)
    with T.Tracer() as tr:
        graph.replay()
        graph.replay()
    ls = check_launches(tr)
    assert [launch.kernel for launch in ls] == ["permute_bf16", "permute_bf16"]
    assert all(launch.ctas == one.ctas for launch in ls)


def test_attach_argument_errors():
    raw = torch.zeros(4096, dtype=torch.uint8, device="cuda")
    count = torch.zeros(1, dtype=torch.int32, device="cuda")
    with pytest.raises(B.MoeError) as e:
        B.moe_trace_attach(raw, None)                  # records without a counter
    assert e.value.code == B.MOE_ERR_INVALID_ARG
    with pytest.raises(B.MoeError) as e:
        B.moe_trace_attach(raw[1:1 + 32 * 8], count)   # records not 8-byte aligned
    assert e.value.code == B.MOE_ERR_INVALID_ARG
    with pytest.raises(B.MoeError) as e:
        B.moe_trace_attach(raw[:16], count)            # capacity 0
    assert e.value.code == B.MOE_ERR_INVALID_ARG
    B.moe_trace_attach(None, None)


def test_next_row_kernels_record_with_their_variants():
    w = make_workload("mid_zipf", n_tokens=512)
    run = GpuRun(w, quant=False, combine=False)
    prob, buf = run.prob, run.buf
    rows, H = buf.rows, w.H
    hidden = to_dev_bf16(w.hidden)
    X = to_dev_bf16(w.expert_out)
    gates = torch.from_numpy(w.gates).cuda()
    gs = torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")
    prob_a = B.Problem(**{**prob.__dict__, "flags": B.MOE_FLAG_NVFP4_SWIZZLED_SCALES})
    atoms = torch.empty(B.nvfp4_swizzled_scale_bytes(rows, H), dtype=torch.uint8,
                        device="cuda")
    I = H // 2
    codes6, scales6 = B.swiglu_buffers(rows, I, B.MOE_QUANT_MXFP6_E2M3)
    codes8, scales8 = B.swiglu_buffers(rows, I, B.MOE_QUANT_MXFP8)
    seg = torch.empty((rows, H), dtype=torch.bfloat16, device="cuda")
    peer = torch.tensor([seg.data_ptr()] * w.S, dtype=torch.int64, device="cuda")
    put = torch.zeros(w.S, dtype=torch.int64, device="cuda")
    bufs8 = (torch.empty((rows, H), dtype=torch.uint8, device="cuda"),
             torch.empty((rows, H // 128), dtype=torch.float32, device="cuda"))
    bufs4 = (torch.empty((rows, H // 2), dtype=torch.uint8, device="cuda"),
             torch.empty((rows, H // 16), dtype=torch.uint8, device="cuda"))
    q8 = [torch.tensor([t.data_ptr()] * w.S, dtype=torch.int64, device="cuda") for t in bufs8]
    q4 = [torch.tensor([t.data_ptr()] * w.S, dtype=torch.int64, device="cuda") for t in bufs4]
    with T.Tracer() as tr:
        B.moe_permute_premultiplied(prob, hidden, buf.row_src, buf.pair_slot, gates, buf.out)
        B.moe_permute_backward(prob, X, buf.pair_slot, poisoned_empty((w.N, H), torch.bfloat16))
        B.moe_combine_backward(prob, hidden, X, gates, buf.pair_slot, buf.row_src,
                               poisoned_empty((rows, H), torch.bfloat16),
                               poisoned_empty((w.N, w.k), torch.float32))
        B.moe_permute_quant_nvfp4(prob_a, hidden, buf.row_src, buf.pair_slot, gs, buf.out_fp4,
                                  atoms)
        B.moe_swiglu_quant(prob, I, B.MOE_QUANT_MXFP8, B.MOE_GATE_UP_SPLIT, X, buf.row_src, gs,
                           codes8, scales8)
        B.moe_swiglu_quant(prob, I, B.MOE_QUANT_MXFP6_E2M3, B.MOE_GATE_UP_SPLIT, X,
                           buf.row_src, gs, codes6, scales6)
        # every segment into the same buffer at offset 0 (each segment fits;
        # only the records matter here)
        B.moe_permute_to_peers(prob, hidden, buf.row_src, buf.pair_slot, buf.meta, peer, put)
        B.moe_permute_quant_fp8_to_peers(prob, hidden, buf.row_src, buf.pair_slot, buf.meta,
                                         *q8, put)
        B.moe_permute_quant_nvfp4_to_peers(prob, hidden, buf.row_src, buf.pair_slot, buf.meta,
                                           gs, *q4, put)
        B.moe_combine_from_peers(prob, peer, put, buf.meta, gates, buf.pair_slot,
                                 poisoned_empty((w.N, H), torch.bfloat16))
    got = [(launch.kernel, launch.variant) for launch in check_launches(tr)]
    nvfp4 = [g for g in got if g[0] in ("permute_nvfp4", "scales_to_atoms")]
    assert got[:3] == [("permute_premultiplied", 0), ("permute_backward", 8),
                       ("combine_backward", 8)]
    assert nvfp4 in ([("permute_nvfp4", 0), ("scales_to_atoms", 1)], [("permute_nvfp4", 1)])
    assert got[-6:] == [("swiglu_split", B.MOE_QUANT_MXFP8),
                        ("swiglu_quant", B.MOE_QUANT_MXFP6_E2M3), ("permute_to_peers", 0),
                        ("permute_fp8_to_peers", 0), ("permute_nvfp4_to_peers", 0),
                        ("combine_from_peers", 8)]
