"""Helpers for the GPU parity tests: run the CUDA path through the C-ABI
binding on a workload and bring every output back as numpy arrays.

Every output buffer is filled with a poison pattern before the library is
called (NaN bit patterns for bf16 and fp32 data, 0xA5 bytes for codes and
scales, -7 for the int32 maps and tables, 9 for the drop mask, all ones for
the status word), so an element a kernel fails to write keeps a value no
correct kernel produces and fails the comparison with the oracle.
"""
from __future__ import annotations

import concurrent.futures as cf
import os

import numpy as np
import torch

from combine_topk_ids_scan_b200 import binding as B

BF16_POISON = 0x7FC1        # a bf16 NaN
F32_POISON = 0x7FA5A5A5     # an fp32 NaN
BYTE_POISON = 0xA5
I32_POISON = -7
MASK_POISON = 9


def poison(t: torch.Tensor | None, value: int | None = None) -> torch.Tensor | None:
    """Fill t (in place) with its dtype's poison pattern (or `value`)."""
    if t is None:
        return t
    if t.dtype == torch.bfloat16:
        t.view(torch.int16).fill_(BF16_POISON if value is None else value)
    elif t.dtype == torch.float32:
        t.view(torch.int32).fill_(F32_POISON if value is None else value)
    elif t.dtype == torch.uint8:
        t.fill_(BYTE_POISON if value is None else value)
    elif t.dtype == torch.int32:
        t.fill_(I32_POISON if value is None else value)
    else:
        raise TypeError(f"no poison for {t.dtype}")
    return t


def poisoned_empty(shape, dtype, device="cuda") -> torch.Tensor:
    return poison(torch.empty(shape, dtype=dtype, device=device))


def poison_buffers(buf: B.Buffers) -> B.Buffers:
    """Poison every output of a Buffers set (the workspace stays zero: the
    layout requires a zero-filled workspace)."""
    for name in ("expert_counts", "expert_offsets", "meta", "row_src", "pair_slot"):
        poison(getattr(buf, name))
    poison(buf.drop_mask, MASK_POISON)
    poison(buf.status, -1)
    for name in ("out", "out_fp8", "scales_fp8", "out_fp4", "scales_fp4", "out_mx4",
                 "scales_mx4"):
        poison(getattr(buf, name, None))
    return buf


def to_dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def bf16_np(t: torch.Tensor) -> np.ndarray:
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def problem_of(w, flags: int = 0, pad: int = 0) -> B.Problem:
    return B.Problem(num_tokens=w.N, hidden=w.H, num_experts=w.E, top_k=w.k,
                     num_segments=w.S, recv_capacity=w.recv_capacity,
                     expert_capacity=w.expert_capacity, flags=flags,
                     expert_pad_multiple=pad)


def par_rows(fn, n: int, *arrays, chunk: int = 4096):
    """fn(*[a[i0:i1] for a in arrays]) over row chunks of [0, n), in threads
    (each oracle call is single-threaded C and releases the GIL); the
    results (an array or a tuple of arrays) are concatenated along axis 0.
    Rows are independent in every function this is used with."""
    bounds = [(i, min(n, i + chunk)) for i in range(0, n, chunk)] or [(0, 0)]
    workers = max(1, min(len(bounds), os.cpu_count() or 1, 32))
    with cf.ThreadPoolExecutor(workers) as ex:
        parts = list(ex.map(lambda b: fn(*[a[b[0]:b[1]] for a in arrays]), bounds))
    if isinstance(parts[0], tuple):
        return tuple(np.concatenate([p[i] for p in parts]) for i in range(len(parts[0])))
    return np.concatenate(parts)


class GpuRun:
    """All outputs of one pass of the CUDA path (layout, the three permutes
    where the shape allows them, combine), every output poisoned first."""

    def __init__(self, w, flags: int = 0, quant: bool = True, combine: bool = True,
                 expert_out: np.ndarray | None = None, pad: int = 0):
        prob = problem_of(w, flags, pad)
        self.prob = prob
        self.swizzled = bool(flags & B.MOE_FLAG_NVFP4_SWIZZLED_SCALES)
        buf = poison_buffers(B.Buffers(prob))
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
            y = poisoned_empty((w.N, w.H), torch.bfloat16)
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
