"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI
binding on a workload and bring every output back as numpy arrays."""
from __future__ import annotations

import numpy as np
import torch

from combine_topk_ids_scan_b200 import binding as B


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def problem_of(w, flags: int = 0, pad: int = 0) -> B.Problem:
    return B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity, flags=flags,
                     expert_pad_multiple=pad)


class GpuRun:
    """All outputs of one pass of the CUDA path (layout, the three permutes
    where the shape allows them, combine)."""

    def __init__(self, w, flags: int = 0, quant: bool = True, combine: bool = True,
                 expert_out: np.ndarray | None = None, pad: int = 0):
        prob = problem_of(w, flags, pad)
        self.prob = prob
        self.swizzled = bool(flags & B.MOE_FLAG_NVFP4_SWIZZLED_SCALES)
        buf = B.Buffers(prob)
        self.buf = buf
        ids = torch.from_numpy(np.ascontiguousarray(w.ids)).cuda()
        B.layout(prob, ids, buf)
        hidden = to_dev_bf16(w.hidden) if w.N > 0 else torch.empty(
            (1, w.H), dtype=torch.bfloat16, device="cuda")
        B.moe_permute(prob, hidden, buf.row_src, buf.pair_slot, buf.out)
        self.has_fp8 = quant and w.H % 128 == 0
        self.has_fp4 = quant and w.H % 32 == 0
        if self.has_fp8:
            B.moe_permute_quant_fp8(prob, hidden, buf.row_src, buf.pair_slot, buf.out_fp8,
                                    buf.scales_fp8)
        if self.has_fp4:
            gs = torch.tensor([w.global_scale], dtype=torch.float32, device="cuda")
            B.moe_permute_quant_nvfp4(prob, hidden, buf.row_src, buf.pair_slot, gs,
                                      buf.out_fp4, buf.scales_fp4)
            B.moe_permute_quant_mxfp4(prob, hidden, buf.row_src, buf.pair_slot, buf.out_mx4,
                                      buf.scales_mx4)
        self.y = None
        if combine and w.N > 0:
            X = expert_out if expert_out is not None else w.expert_out
            Xd = to_dev_bf16(X)
            gates = torch.from_numpy(np.ascontiguousarray(w.gates)).cuda()
            y = torch.empty((w.N, w.H), dtype=torch.bfloat16, device="cuda")
            B.moe_combine(prob, Xd, gates, buf.pair_slot, y)
            self.y_dev = y
        torch.cuda.synchronize()
        rows = buf.rows
        N = w.N
        self.status = int(buf.status.cpu().numpy().view(np.uint32)[0])
        self.expert_counts = buf.expert_counts.cpu().numpy()
        self.expert_offsets = buf.expert_offsets.cpu().numpy()
        self.meta = buf.meta.cpu().numpy().view(np.uint32)
        self.row_src = buf.row_src.cpu().numpy()[:rows]
        self.pair_slot = buf.pair_slot.cpu().numpy()[:N]
        self.drop_mask = buf.drop_mask.cpu().numpy()[:N]
        self.out = bf16_np(buf.out)[:rows]
        if self.has_fp8:
            self.q8 = buf.out_fp8.cpu().numpy()[:rows]
            self.s8 = buf.scales_fp8.cpu().numpy()[:rows]
        if self.has_fp4:
            self.q4 = buf.out_fp4.cpu().numpy()[:rows]
            self.qmx = buf.out_mx4.cpu().numpy()[:rows]
            if flags & B.MOE_FLAG_NVFP4_SWIZZLED_SCALES:
                self.s4 = buf.scales_fp4.cpu().numpy().reshape(-1)   # atom layout, flat
                self.smx = buf.scales_mx4.cpu().numpy().reshape(-1)
            else:
                self.s4 = buf.scales_fp4.cpu().numpy()[:rows]
                self.smx = buf.scales_mx4.cpu().numpy()[:rows]
        if combine and w.N > 0:
            self.y = bf16_np(self.y_dev)
