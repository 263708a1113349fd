"""The largest output the library accepts: rows * H just below 2^32 elements
(the [4, S] table counts elements in uint32), so byte offsets of the bf16
rows and of the combine's expert rows run to nearly 8 GiB, past 4 GiB, and
every kernel's 64-bit address arithmetic is exercised.  N = 131071 tokens, H = 4096,
E = 256, k = 8, rows = 2^20 - 1 (seven padding rows); P = 1,048,568 pairs
takes the scan + emit layout kernels.

Outputs this large are compared on samples the oracle computes one by one:
the layout in full; 4096 random rows plus the first and last 16 of every
permute output (bf16, FP8, NVFP4, MXFP4); 2048 random tokens plus the last
16 of the combine, the oracle given exactly the expert rows those tokens
read.  Every output buffer is poisoned first."""
import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200.inputs import normal_bf16, softmax_gates
from gpu_util import bf16_np, poison_buffers, poisoned_empty, to_dev_bf16

pytestmark = pytest.mark.gpu

N, H, E, K, S = 131071, 4096, 256, 8, 8
ROWS = (1 << 20) - 1


@pytest.fixture(scope="module", autouse=True)
def _need_gpu():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    build.build()
    B.load()


def _sample(n, count, rng):
    s = set(rng.choice(n, size=min(count, n), replace=False).tolist())
    s |= set(range(min(16, n))) | set(range(max(0, n - 16), n))
    return np.array(sorted(s), dtype=np.int64)


def test_maximum_element_count(orc):
    assert ROWS * H < 1 << 32 and ROWS * H * 2 > 1 << 32   # bf16 byte offsets past 4 GiB
    ss = np.random.SeedSequence(4242)
    s_ids, s_hid, s_gate, s_pick = ss.spawn(4)
    rng = np.random.Generator(np.random.PCG64(s_ids))
    ids = np.argsort(rng.random((N, E), dtype=np.float32), axis=1)[:, :K].astype(np.int32)
    hidden = normal_bf16(s_hid, N, H)
    gates = softmax_gates(np.random.Generator(np.random.PCG64(s_gate)), N, K)

    prob = B.Problem(num_tokens=N, hidden=H, num_experts=E, top_k=K, num_segments=S,
                     recv_capacity=ROWS)
    buf = poison_buffers(B.Buffers(prob))
    d_hidden = to_dev_bf16(hidden)
    # the global scale amax / 2688 (the maximum of bf16 values is exact)
    gs_val = float(np.float32(d_hidden.abs().max().float().item()) / np.float32(2688.0))
    gs = torch.tensor([gs_val], dtype=torch.float32, device="cuda")
    B.layout(prob, torch.from_numpy(ids).cuda(), buf)
    B.moe_permute(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out)
    B.moe_permute_quant_fp8(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out_fp8,
                            buf.scales_fp8)
    B.moe_permute_quant_nvfp4(prob, d_hidden, buf.row_src, buf.pair_slot, gs, buf.out_fp4,
                              buf.scales_fp4)
    B.moe_permute_quant_mxfp4(prob, d_hidden, buf.row_src, buf.pair_slot, buf.out_mx4,
                              buf.scales_mx4)
    # expert outputs [ROWS, H] bf16 drawn on the device (seeded), in chunks
    gen = torch.Generator(device="cuda")
    gen.manual_seed(99)
    X = torch.empty((ROWS, H), dtype=torch.bfloat16, device="cuda")
    for r0 in range(0, ROWS, 1 << 17):
        r1 = min(ROWS, r0 + (1 << 17))
        X[r0:r1] = torch.randn((r1 - r0, H), generator=gen, device="cuda").to(torch.bfloat16)
    y = poisoned_empty((N, H), torch.bfloat16)
    B.moe_combine(prob, X, torch.from_numpy(gates).cuda(), buf.pair_slot, y)
    torch.cuda.synchronize()

    # layout, in full
    ref = orc.layout(ids, E, S, H, recv_capacity=ROWS)
    assert int(buf.status.item()) == ref.status == 0
    assert np.array_equal(buf.expert_counts.cpu().numpy(), ref.expert_counts)
    assert np.array_equal(buf.expert_offsets.cpu().numpy(), ref.expert_offsets)
    assert np.array_equal(buf.meta.cpu().numpy().view(np.uint32), ref.meta)
    assert np.array_equal(buf.row_src.cpu().numpy()[:ROWS], ref.row_src)
    assert np.array_equal(buf.pair_slot.cpu().numpy()[:N], ref.pair_slot)

    # permute outputs on sampled rows
    pick = np.random.Generator(np.random.PCG64(s_pick))
    rows = _sample(ROWS, 4096, pick)
    ri = torch.from_numpy(rows).cuda()
    rs = ref.row_src[rows]

    def take(t):
        return t.index_select(0, ri).cpu().numpy()

    assert np.array_equal(take(buf.out.view(torch.int16)).view(np.uint16),
                          orc.permute_bf16(hidden, rs))
    q, sc = orc.permute_fp8(hidden, rs)
    assert np.array_equal(take(buf.out_fp8), q)
    assert np.array_equal(take(buf.scales_fp8).view(np.uint32), sc.view(np.uint32))
    q, sc = orc.permute_nvfp4(hidden, rs, gs_val)
    assert np.array_equal(take(buf.out_fp4), q)
    assert np.array_equal(take(buf.scales_fp4), sc)
    q, sc = orc.permute_mxfp4(hidden, rs)
    assert np.array_equal(take(buf.out_mx4), q)
    assert np.array_equal(take(buf.scales_mx4), sc)

    # combine on sampled tokens: the oracle gets exactly the rows they read
    toks = _sample(N, 2048, pick)
    slots = ref.pair_slot[toks]                                   # [T, K]
    used = np.unique(slots[slots >= 0])
    x_sub = bf16_np(X.index_select(0, torch.from_numpy(used).cuda()))
    remap = np.full(ROWS, -1, np.int64)
    remap[used] = np.arange(used.size)
    slots_sub = np.where(slots >= 0, remap[np.maximum(slots, 0)], -1).astype(np.int32)
    want = orc.combine(x_sub, np.ascontiguousarray(gates[toks]), slots_sub)
    got = bf16_np(y.index_select(0, torch.from_numpy(toks).cuda()))
    assert np.array_equal(got, want)
