"""GPU parity of the dispatch with pre-multiplied gates
(moe_permute_premultiplied) against the oracle, bit for bit: packed and
capacity layouts, padding rows, masked, out-of-range and dropped pairs, a
ragged last chunk (H not a multiple of 512), top_k 1 and 16, every row
masked.  Kept in its own file, after the other GPU tests."""
import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200.inputs import make_workload
from gpu_util import GpuRun, bf16_np, to_dev_bf16
from test_gpu_parity import custom, oracle_layout

pytestmark = pytest.mark.gpu

CASES = {
    "tiny": lambda: make_workload("tiny"),
    "decode_capacity": lambda: make_workload("decode_capacity"),
    "padded_masked_badids": lambda: custom(N=333, H=200, E=12, k=3, S=4, C=1100, p_mask=0.1,
                                           p_bad=0.02, seed=5),
    "k16_ragged": lambda: custom(N=100, H=1088, E=64, k=16, S=16, seed=6),
    "k1": lambda: custom(N=700, H=96, E=7, k=1, S=7, seed=7),
    "all_masked": lambda: custom(N=64, H=128, E=4, k=2, S=1, C=40, p_mask=1.1, seed=8),
    "capacity_drops": lambda: custom(N=900, H=256, E=32, k=4, S=8, Ce=3, seed=9),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_permute_premultiplied_parity(orc, name):
    w = CASES[name]()
    run = GpuRun(w, quant=False, combine=False)
    ref = oracle_layout(orc, w)
    assert np.array_equal(run.pair_slot, ref.pair_slot)
    rows = run.buf.rows
    hidden = to_dev_bf16(w.hidden)
    gates = torch.from_numpy(np.ascontiguousarray(w.gates)).cuda()
    out = torch.full((max(rows, 1), w.H), float("nan"), dtype=torch.bfloat16, device="cuda")
    B.moe_permute_premultiplied(run.prob, hidden, run.buf.row_src, run.buf.pair_slot, gates, out)
    torch.cuda.synchronize()
    want = orc.permute_premultiplied(w.hidden, w.gates, ref.pair_slot, rows)
    assert np.array_equal(bf16_np(out)[:rows], want)
