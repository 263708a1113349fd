"""Thin ctypes binding of libmoedc.so (declared in include/moe_dc.h).

Each function has the name of the C entry point it calls and only marshals
arguments: torch tensors become device pointers, the current torch CUDA
stream becomes the launch stream.  Every step of the computation runs in the
library's CUDA kernels; there is no fallback of any kind -- if the library
cannot be loaded, the first call raises.

The C ABI takes plain pointers and cannot see buffer sizes, so before a call
each function checks that every tensor it passes holds at least the bytes
the problem needs (moe_dc.h gives each array's shape) and raises
MoeError(MOE_ERR_INVALID_ARG) otherwise: a short buffer becomes a Python
error instead of an out-of-bounds device access.
"""
from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
# MOE_LIB_PATH selects another build of the library, e.g. the build with
# device index checks (libmoedc_debug.so, see moe_debug_violations) or the
# build with trace records
LIB_PATH = os.environ.get("MOE_LIB_PATH") or os.path.join(_PKG, "libmoedc.so")
DEBUG_LIB_PATH = os.path.join(_PKG, "libmoedc_debug.so")
# per-CTA trace records (libmoedc_trace.so, see moe_trace_attach)
TRACE_LIB_PATH = os.path.join(_PKG, "libmoedc_trace.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED_SHAPE = 2
MOE_ERR_CUDA = 3
MOE_ERR_NOT_BUILT = 4

MOE_STATUS_ID_RANGE = 1
MOE_STATUS_DUP_ID = 2
MOE_STATUS_CAPACITY = 4
MOE_STATUS_TIMEOUT = 8

MOE_FLAG_CHECK_DUPLICATES = 1
MOE_FLAG_LAYOUT_TWO_PASS = 2
MOE_FLAG_NVFP4_SWIZZLED_SCALES = 4
MOE_FLAG_LAYOUT_LOOKBACK = 8
MOE_FLAG_TEST_STALL_SCAN = 0x80000000

MOE_MAX_EXPERTS = 2048
MOE_MAX_TOPK = 16

# every symbol include/moe_dc.h declares
EXPORTED = ("moe_output_rows", "moe_workspace_bytes", "moe_dispatch_layout",
            "moe_dispatch_layout_noalloc", "moe_permute", "moe_permute_premultiplied",
            "moe_permute_to_peers", "moe_permute_quant_fp8_to_peers",
            "moe_permute_quant_nvfp4_to_peers", "moe_combine_from_peers",
            "moe_permute_quant_fp8",
            "moe_permute_quant_nvfp4", "moe_permute_quant_mxfp4", "moe_combine",
            "moe_permute_backward",
            "moe_combine_backward", "moe_swiglu_quant", "moe_status_string", "moe_version",
            "moe_debug_violations", "moe_trace_attach")

(MOE_QUANT_NVFP4, MOE_QUANT_MXFP8, MOE_QUANT_MXFP4, MOE_QUANT_BF16, MOE_QUANT_MXFP6_E2M3,
 MOE_QUANT_MXFP6_E3M2) = 0, 1, 2, 3, 4, 5
MOE_GATE_UP_SPLIT, MOE_GATE_UP_INTERLEAVED = 0, 1

MOE_NOALLOC_SCRATCH_BYTES = 1 << 20


_STATUS_TEXT = {MOE_OK: "ok", MOE_ERR_INVALID_ARG: "invalid argument",
                MOE_ERR_UNSUPPORTED_SHAPE: "unsupported shape", MOE_ERR_CUDA: "CUDA error",
                MOE_ERR_NOT_BUILT: "not in this build"}


class MoeError(RuntimeError):
    def __init__(self, code: int, where: str):
        try:
            text = status_string(code)
        except Exception:            # the library's own text when it can be loaded
            text = _STATUS_TEXT.get(code, "unknown status")
        super().__init__(f"{where}: {text} (moe_status {code})")
        self.code = code


class moe_problem(ctypes.Structure):
    _fields_ = [("num_tokens", ctypes.c_int32), ("hidden", ctypes.c_int32),
                ("num_experts", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("num_segments", ctypes.c_int32), ("expert_capacity", ctypes.c_int32),
                ("recv_capacity", ctypes.c_int64), ("flags", ctypes.c_uint32),
                ("expert_pad_multiple", ctypes.c_int32)]


@dataclass
class Problem:
    """Sizes of one dispatch / combine problem (see moe_problem in moe_dc.h)."""
    num_tokens: int
    hidden: int
    num_experts: int
    top_k: int
    num_segments: int = 1
    recv_capacity: int = 0
    expert_capacity: int = 0
    flags: int = 0
    expert_pad_multiple: int = 0

    def c(self) -> moe_problem:
        return moe_problem(self.num_tokens, self.hidden, self.num_experts, self.top_k,
                           self.num_segments, self.expert_capacity, self.recv_capacity,
                           self.flags & 0xFFFFFFFF, self.expert_pad_multiple)


_lib = None


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libmoedc.so (once).  Raises if it is missing: there is no
    fallback path."""
    global _lib
    if _lib is not None:
        return _lib
    path = path or LIB_PATH
    if not os.path.exists(path):
        raise RuntimeError(f"libmoedc.so not found at {path}; build it with "
                           "`python -m combine_topk_ids_scan_b200.build`")
    L = ctypes.CDLL(path)
    vp, P = ctypes.c_void_p, ctypes.POINTER(moe_problem)
    L.moe_output_rows.restype = ctypes.c_int64
    L.moe_output_rows.argtypes = [P]
    L.moe_workspace_bytes.restype = ctypes.c_size_t
    L.moe_workspace_bytes.argtypes = [P]
    L.moe_dispatch_layout.restype = ctypes.c_int
    L.moe_dispatch_layout.argtypes = [P] + [vp] * 10
    L.moe_dispatch_layout_noalloc.restype = ctypes.c_int
    L.moe_dispatch_layout_noalloc.argtypes = [P] + [vp] * 9
    L.moe_permute.restype = ctypes.c_int
    L.moe_permute.argtypes = [P] + [vp] * 5
    L.moe_permute_to_peers.restype = ctypes.c_int
    L.moe_permute_to_peers.argtypes = [P] + [vp] * 7
    L.moe_permute_quant_fp8_to_peers.restype = ctypes.c_int
    L.moe_permute_quant_fp8_to_peers.argtypes = [P] + [vp] * 8
    L.moe_permute_quant_nvfp4_to_peers.restype = ctypes.c_int
    L.moe_permute_quant_nvfp4_to_peers.argtypes = [P] + [vp] * 9
    L.moe_combine_from_peers.restype = ctypes.c_int
    L.moe_combine_from_peers.argtypes = [P] + [vp] * 7
    L.moe_permute_premultiplied.restype = ctypes.c_int
    L.moe_permute_premultiplied.argtypes = [P] + [vp] * 6
    L.moe_permute_quant_fp8.restype = ctypes.c_int
    L.moe_permute_quant_fp8.argtypes = [P] + [vp] * 6
    L.moe_permute_quant_nvfp4.restype = ctypes.c_int
    L.moe_permute_quant_nvfp4.argtypes = [P] + [vp] * 7
    L.moe_permute_quant_mxfp4.restype = ctypes.c_int
    L.moe_permute_quant_mxfp4.argtypes = [P] + [vp] * 6
    L.moe_combine.restype = ctypes.c_int
    L.moe_combine.argtypes = [P] + [vp] * 5
    L.moe_permute_backward.restype = ctypes.c_int
    L.moe_permute_backward.argtypes = [P] + [vp] * 4
    L.moe_combine_backward.restype = ctypes.c_int
    L.moe_combine_backward.argtypes = [P] + [vp] * 8
    L.moe_swiglu_quant.restype = ctypes.c_int
    L.moe_swiglu_quant.argtypes = [P, ctypes.c_int32, ctypes.c_uint32, ctypes.c_uint32] + \
        [vp] * 6
    L.moe_status_string.restype = ctypes.c_char_p
    L.moe_status_string.argtypes = [ctypes.c_int]
    L.moe_version.restype = ctypes.c_char_p
    L.moe_version.argtypes = []
    L.moe_debug_violations.restype = ctypes.c_int64
    L.moe_debug_violations.argtypes = [ctypes.c_int]
    L.moe_trace_attach.restype = ctypes.c_int
    L.moe_trace_attach.argtypes = [vp, ctypes.c_uint32, vp, vp]
    _lib = L
    return L


def status_string(code: int) -> str:
    return load().moe_status_string(code).decode()


def version() -> str:
    return load().moe_version().decode()


def debug_violations(reset: bool = False) -> int:
    """Bits of out-of-range indices the device checks recorded (0 = none),
    or -1 when the loaded build has no checks (see moe_debug_violations)."""
    return int(load().moe_debug_violations(int(reset)))


TRACE_RECORD_BYTES = 32   # sizeof(moe_trace_record)


def moe_trace_attach(records, count, stream=None) -> None:
    """Attach a trace record buffer (the build with -DMOE_TRACE): `records`
    is a device tensor of capacity * 32 bytes, `count` a device int32 tensor
    of at least one element that the caller has zeroed; records=None
    detaches.  Raises MoeError(MOE_ERR_NOT_BUILT) on other builds."""
    if records is None:
        _check(load().moe_trace_attach(None, 0, None, _stream(stream)), "moe_trace_attach")
        return
    capacity = records.numel() * records.element_size() // TRACE_RECORD_BYTES
    _require("moe_trace_attach", count=(count, 4))
    _check(load().moe_trace_attach(_ptr(records), capacity, _ptr(count), _stream(stream)),
           "moe_trace_attach")


def _ptr(t: torch.Tensor | None):
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("expected a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError("expected a contiguous tensor")
    return ctypes.c_void_p(t.data_ptr())


def _sizes(prob: Problem):
    """(N, H, E, k, S, P, rows) of a problem, negatives clamped to 0 (an
    invalid problem is then rejected by the library itself)."""
    N, H, E, k, S = (max(0, int(v)) for v in (prob.num_tokens, prob.hidden, prob.num_experts,
                                                prob.top_k, prob.num_segments))
    rows = E * max(0, prob.expert_capacity) if prob.expert_capacity > 0 \
        else max(0, int(prob.recv_capacity))
    return N, H, E, k, S, N * k, rows


def _require(where: str, **need) -> None:
    """need: argument name -> (tensor or None, bytes the problem needs).
    Raises MoeError(MOE_ERR_INVALID_ARG) for a tensor holding fewer bytes;
    None (the library checks which pointers may be null) and zero-byte needs
    are skipped."""
    for name, (t, nbytes) in need.items():
        if t is None or nbytes <= 0:
            continue
        have = t.numel() * t.element_size()
        if have < nbytes:
            raise MoeError(MOE_ERR_INVALID_ARG,
                           f"{where}: {name} holds {have} bytes, the problem needs {nbytes}")


def _stream(stream: torch.cuda.Stream | None):
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def _check(code: int, where: str) -> None:
    if code != MOE_OK:
        raise MoeError(code, where)


def moe_output_rows(prob: Problem) -> int:
    return int(load().moe_output_rows(ctypes.byref(prob.c())))


def moe_workspace_bytes(prob: Problem) -> int:
    return int(load().moe_workspace_bytes(ctypes.byref(prob.c())))


def _layout_need(prob: Problem, topk_ids, expert_counts, expert_offsets, meta, row_src,
                 pair_slot, drop_mask, status) -> dict:
    N, H, E, k, S, P, rows = _sizes(prob)
    return dict(topk_ids=(topk_ids, 4 * P), expert_counts=(expert_counts, 4 * E),
                expert_offsets=(expert_offsets, 4 * (E + 1)), meta=(meta, 16 * S),
                row_src=(row_src, 4 * rows), pair_slot=(pair_slot, 4 * P),
                drop_mask=(drop_mask, P), status=(status, 4))


def moe_dispatch_layout(prob: Problem, topk_ids, expert_counts, expert_offsets, meta, row_src,
                        pair_slot, drop_mask, status, workspace, stream=None) -> None:
    _require("moe_dispatch_layout",
             **_layout_need(prob, topk_ids, expert_counts, expert_offsets, meta, row_src,
                            pair_slot, drop_mask, status),
             workspace=(workspace, moe_workspace_bytes(prob)))
    c = prob.c()
    _check(load().moe_dispatch_layout(ctypes.byref(c), _ptr(topk_ids), _ptr(expert_counts),
                                      _ptr(expert_offsets), _ptr(meta), _ptr(row_src),
                                      _ptr(pair_slot), _ptr(drop_mask), _ptr(status),
                                      _ptr(workspace), _stream(stream)),
           "moe_dispatch_layout")


def moe_dispatch_layout_noalloc(prob: Problem, topk_ids, expert_counts, expert_offsets, meta,
                                row_src, pair_slot, drop_mask, status, stream=None) -> None:
    """The layout without a caller workspace (for callers that cannot
    allocate); see moe_dispatch_layout_noalloc in moe_dc.h for its limits."""
    _require("moe_dispatch_layout_noalloc",
             **_layout_need(prob, topk_ids, expert_counts, expert_offsets, meta, row_src,
                            pair_slot, drop_mask, status))
    c = prob.c()
    _check(load().moe_dispatch_layout_noalloc(ctypes.byref(c), _ptr(topk_ids),
                                              _ptr(expert_counts), _ptr(expert_offsets),
                                              _ptr(meta), _ptr(row_src), _ptr(pair_slot),
                                              _ptr(drop_mask), _ptr(status), _stream(stream)),
           "moe_dispatch_layout_noalloc")


def _permute_need(prob: Problem, hidden_states, row_src, pair_slot) -> dict:
    N, H, E, k, S, P, rows = _sizes(prob)
    return dict(hidden_states=(hidden_states, 2 * N * H), row_src=(row_src, 4 * rows),
                pair_slot=(pair_slot, 4 * P))


def moe_permute(prob: Problem, hidden_states, row_src, pair_slot, out, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute", **_permute_need(prob, hidden_states, row_src, pair_slot),
             out=(out, 2 * rows * H))
    c = prob.c()
    _check(load().moe_permute(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                              _ptr(pair_slot), _ptr(out), _stream(stream)), "moe_permute")


def moe_permute_to_peers(prob: Problem, hidden_states, row_src, pair_slot, meta, peer_out,
                         put_offsets, stream=None) -> None:
    """Dispatch permute whose segment s lands in rank s's receive buffer:
    peer_out is an int64 device tensor of S device addresses (e.g.
    [t.data_ptr() for t in receive buffers]), put_offsets an int64 device
    tensor of S first rows (see moe_permute_to_peers in moe_dc.h).  The
    library sees only the addresses: that every receive buffer holds its
    rows is the caller's to guarantee."""
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_to_peers", **_permute_need(prob, hidden_states, row_src, pair_slot),
             meta=(meta, 16 * S), peer_out=(peer_out, 8 * S), put_offsets=(put_offsets, 8 * S))
    c = prob.c()
    _check(load().moe_permute_to_peers(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                                       _ptr(pair_slot), _ptr(meta), _ptr(peer_out),
                                       _ptr(put_offsets), _stream(stream)),
           "moe_permute_to_peers")


def moe_permute_quant_fp8_to_peers(prob: Problem, hidden_states, row_src, pair_slot, meta,
                                   peer_codes, peer_scales, put_offsets, stream=None) -> None:
    """FP8 dispatch whose segment s lands in rank s's receive buffers:
    peer_codes / peer_scales are int64 device tensors of S device addresses
    (E4M3 [rows, H] and fp32 [rows, H/128] buffers), put_offsets as in
    moe_permute_to_peers (see moe_permute_quant_fp8_to_peers in moe_dc.h);
    the receive buffers' sizes are the caller's to guarantee."""
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_quant_fp8_to_peers",
             **_permute_need(prob, hidden_states, row_src, pair_slot), meta=(meta, 16 * S),
             peer_codes=(peer_codes, 8 * S), peer_scales=(peer_scales, 8 * S),
             put_offsets=(put_offsets, 8 * S))
    c = prob.c()
    _check(load().moe_permute_quant_fp8_to_peers(
        ctypes.byref(c), _ptr(hidden_states), _ptr(row_src), _ptr(pair_slot), _ptr(meta),
        _ptr(peer_codes), _ptr(peer_scales), _ptr(put_offsets), _stream(stream)),
        "moe_permute_quant_fp8_to_peers")


def moe_permute_quant_nvfp4_to_peers(prob: Problem, hidden_states, row_src, pair_slot, meta,
                                     global_scale, peer_codes, peer_scales, put_offsets,
                                     stream=None) -> None:
    """NVFP4 dispatch whose segment s lands in rank s's receive buffers
    (E2M1 [rows, H/2] codes, E4M3 [rows, H/16] row-major scales); see
    moe_permute_quant_nvfp4_to_peers in moe_dc.h; the receive buffers' sizes
    are the caller's to guarantee."""
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_quant_nvfp4_to_peers",
             **_permute_need(prob, hidden_states, row_src, pair_slot), meta=(meta, 16 * S),
             global_scale=(global_scale, 4 if rows > 0 else 0),
             peer_codes=(peer_codes, 8 * S), peer_scales=(peer_scales, 8 * S),
             put_offsets=(put_offsets, 8 * S))
    c = prob.c()
    _check(load().moe_permute_quant_nvfp4_to_peers(
        ctypes.byref(c), _ptr(hidden_states), _ptr(row_src), _ptr(pair_slot), _ptr(meta),
        _ptr(global_scale), _ptr(peer_codes), _ptr(peer_scales), _ptr(put_offsets),
        _stream(stream)), "moe_permute_quant_nvfp4_to_peers")


def moe_permute_premultiplied(prob: Problem, hidden_states, row_src, pair_slot, gates, out,
                              stream=None) -> None:
    """Dispatch with pre-multiplied gates: each pair's row is its token
    scaled by its gate (see moe_permute_premultiplied in moe_dc.h)."""
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_premultiplied",
             **_permute_need(prob, hidden_states, row_src, pair_slot), gates=(gates, 4 * P),
             out=(out, 2 * rows * H))
    c = prob.c()
    _check(load().moe_permute_premultiplied(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                                            _ptr(pair_slot), _ptr(gates), _ptr(out),
                                            _stream(stream)), "moe_permute_premultiplied")


def moe_permute_quant_fp8(prob: Problem, hidden_states, row_src, pair_slot, out_e4m3, scales,
                          stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_quant_fp8", **_permute_need(prob, hidden_states, row_src, pair_slot),
             out_e4m3=(out_e4m3, rows * H), scales=(scales, 4 * rows * (H // 128)))
    c = prob.c()
    _check(load().moe_permute_quant_fp8(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                                        _ptr(pair_slot), _ptr(out_e4m3), _ptr(scales),
                                        _stream(stream)), "moe_permute_quant_fp8")


def _fp4_scale_bytes(prob: Problem, rows: int, H: int, block: int) -> int:
    if prob.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES:
        return nvfp4_swizzled_scale_bytes(rows, H, block) if rows > 0 else 0
    return rows * (H // block)


def moe_permute_quant_nvfp4(prob: Problem, hidden_states, row_src, pair_slot, global_scale,
                            out_e2m1, scales_e4m3, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_quant_nvfp4", **_permute_need(prob, hidden_states, row_src, pair_slot),
             global_scale=(global_scale, 4 if rows > 0 else 0), out_e2m1=(out_e2m1, rows * H // 2),
             scales_e4m3=(scales_e4m3, _fp4_scale_bytes(prob, rows, H, 16)))
    c = prob.c()
    _check(load().moe_permute_quant_nvfp4(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                                          _ptr(pair_slot), _ptr(global_scale), _ptr(out_e2m1),
                                          _ptr(scales_e4m3), _stream(stream)),
           "moe_permute_quant_nvfp4")


def moe_permute_quant_mxfp4(prob: Problem, hidden_states, row_src, pair_slot, out_e2m1,
                            scales_e8m0, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_quant_mxfp4", **_permute_need(prob, hidden_states, row_src, pair_slot),
             out_e2m1=(out_e2m1, rows * H // 2),
             scales_e8m0=(scales_e8m0, _fp4_scale_bytes(prob, rows, H, 32)))
    c = prob.c()
    _check(load().moe_permute_quant_mxfp4(ctypes.byref(c), _ptr(hidden_states), _ptr(row_src),
                                          _ptr(pair_slot), _ptr(out_e2m1), _ptr(scales_e8m0),
                                          _stream(stream)),
           "moe_permute_quant_mxfp4")


def moe_combine(prob: Problem, expert_out, gates, pair_slot, out, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_combine", expert_out=(expert_out, 2 * rows * H if N > 0 else 0),
             gates=(gates, 4 * P), pair_slot=(pair_slot, 4 * P), out=(out, 2 * N * H))
    c = prob.c()
    _check(load().moe_combine(ctypes.byref(c), _ptr(expert_out), _ptr(gates), _ptr(pair_slot),
                              _ptr(out), _stream(stream)), "moe_combine")


def nvfp4_swizzled_scale_bytes(rows: int, hidden: int, block: int = 16) -> int:
    """Bytes of FP4 block scales (block 16: NVFP4, 32: MXFP4) in the 128x4
    atom layout (see moe_dc.h)."""
    return max(1, -(-rows // 128) * 128 * (-(-(hidden // block) // 4) * 4))


def moe_combine_from_peers(prob: Problem, peer_expert_out, get_offsets, meta, gates, pair_slot,
                           out, stream=None) -> None:
    """Combine reading each expert output from the rank that computed it:
    peer_expert_out is an int64 device tensor of S device addresses (bf16
    [*, H] expert-output buffers), get_offsets an int64 device tensor of S
    first rows (see moe_combine_from_peers in moe_dc.h); the buffers' sizes
    are the caller's to guarantee."""
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_combine_from_peers", peer_expert_out=(peer_expert_out, 8 * S),
             get_offsets=(get_offsets, 8 * S), meta=(meta, 16 * S), gates=(gates, 4 * P),
             pair_slot=(pair_slot, 4 * P), out=(out, 2 * N * H))
    c = prob.c()
    _check(load().moe_combine_from_peers(ctypes.byref(c), _ptr(peer_expert_out),
                                         _ptr(get_offsets), _ptr(meta), _ptr(gates),
                                         _ptr(pair_slot), _ptr(out), _stream(stream)),
           "moe_combine_from_peers")


def moe_permute_backward(prob: Problem, grad_out, pair_slot, grad_hidden, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_permute_backward", grad_out=(grad_out, 2 * rows * H if N > 0 else 0),
             pair_slot=(pair_slot, 4 * P), grad_hidden=(grad_hidden, 2 * N * H))
    c = prob.c()
    _check(load().moe_permute_backward(ctypes.byref(c), _ptr(grad_out), _ptr(pair_slot),
                                       _ptr(grad_hidden), _stream(stream)),
           "moe_permute_backward")


def moe_combine_backward(prob: Problem, grad_y, expert_out, gates, pair_slot, row_src,
                         grad_expert_out, grad_gates, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    _require("moe_combine_backward", grad_y=(grad_y, 2 * N * H),
             expert_out=(expert_out, 2 * rows * H), gates=(gates, 4 * P),
             pair_slot=(pair_slot, 4 * P), row_src=(row_src, 4 * rows),
             grad_expert_out=(grad_expert_out, 2 * rows * H), grad_gates=(grad_gates, 4 * P))
    c = prob.c()
    _check(load().moe_combine_backward(ctypes.byref(c), _ptr(grad_y), _ptr(expert_out),
                                       _ptr(gates), _ptr(pair_slot), _ptr(row_src),
                                       _ptr(grad_expert_out), _ptr(grad_gates),
                                       _stream(stream)), "moe_combine_backward")


_SWIGLU_CODE_BYTES = {MOE_QUANT_NVFP4: (1, 2), MOE_QUANT_MXFP8: (1, 1),
                      MOE_QUANT_MXFP4: (1, 2), MOE_QUANT_BF16: (2, 1),
                      MOE_QUANT_MXFP6_E2M3: (3, 4), MOE_QUANT_MXFP6_E3M2: (3, 4)}


def moe_swiglu_quant(prob: Problem, intermediate: int, fmt: int, gate_up_layout: int, gate_up,
                     row_src, global_scale, codes, scales, stream=None) -> None:
    N, H, E, k, S, P, rows = _sizes(prob)
    I = max(0, int(intermediate))
    if fmt in _SWIGLU_CODE_BYTES:         # an unknown format is rejected by the library
        num, den = _SWIGLU_CODE_BYTES[fmt]
        scale_bytes = 0 if fmt == MOE_QUANT_BF16 else I // (16 if fmt == MOE_QUANT_NVFP4 else 32)
        _require("moe_swiglu_quant", gate_up=(gate_up, 4 * rows * I),
                 row_src=(row_src, 4 * rows), codes=(codes, rows * I * num // den),
                 scales=(scales, rows * scale_bytes),
                 global_scale=(global_scale, 4 if fmt == MOE_QUANT_NVFP4 and rows > 0 else 0))
    c = prob.c()
    _check(load().moe_swiglu_quant(ctypes.byref(c), intermediate, fmt, gate_up_layout,
                                   _ptr(gate_up), _ptr(row_src), _ptr(global_scale), _ptr(codes),
                                   _ptr(scales), _stream(stream)), "moe_swiglu_quant")


def swiglu_buffers(rows: int, intermediate: int, fmt: int, device="cuda"):
    """(codes, scales) uint8 device buffers for moe_swiglu_quant."""
    I = intermediate
    code_bytes = {MOE_QUANT_NVFP4: I // 2, MOE_QUANT_MXFP8: I, MOE_QUANT_MXFP4: I // 2,
                  MOE_QUANT_BF16: 2 * I, MOE_QUANT_MXFP6_E2M3: 3 * I // 4,
                  MOE_QUANT_MXFP6_E3M2: 3 * I // 4}[fmt]
    scale_bytes = I // 16 if fmt == MOE_QUANT_NVFP4 else 0 if fmt == MOE_QUANT_BF16 else I // 32
    codes = torch.empty((max(rows, 1), code_bytes), dtype=torch.uint8, device=device)
    scales = torch.empty((max(rows, 1), max(scale_bytes, 1)), dtype=torch.uint8, device=device)
    return codes, scales


# ----------------------------------------------------------------- buffers
class Buffers:
    """Device buffers for one problem (allocated by torch; the library itself
    allocates nothing).  Convenience for callers and tests."""

    def __init__(self, prob: Problem, device="cuda", quant: bool = True):
        N, H, E, k, S = (prob.num_tokens, prob.hidden, prob.num_experts, prob.top_k,
                         prob.num_segments)
        rows = moe_output_rows(prob)
        if rows < 0:
            raise MoeError(MOE_ERR_INVALID_ARG, "Buffers")
        i32, u8 = torch.int32, torch.uint8
        self.rows = rows
        self.expert_counts = torch.empty(E, dtype=i32, device=device)
        self.expert_offsets = torch.empty(E + 1, dtype=i32, device=device)
        self.meta = torch.empty((4, S), dtype=torch.int32, device=device)  # uint32 bits
        self.row_src = torch.empty(max(rows, 1), dtype=i32, device=device)
        self.pair_slot = torch.empty((max(N, 1), k), dtype=i32, device=device)
        self.drop_mask = torch.empty((max(N, 1), k), dtype=u8, device=device)
        self.status = torch.zeros(1, dtype=torch.int32, device=device)
        self.workspace = torch.zeros(max(moe_workspace_bytes(prob), 16), dtype=u8, device=device)
        self.out = torch.empty((max(rows, 1), H), dtype=torch.bfloat16, device=device)
        if quant:
            self.out_fp8 = torch.empty((max(rows, 1), H), dtype=u8, device=device)
            self.scales_fp8 = torch.empty((max(rows, 1), max(H // 128, 1)), dtype=torch.float32,
                                          device=device)
            self.out_fp4 = torch.empty((max(rows, 1), H // 2), dtype=u8, device=device)
            if prob.flags & MOE_FLAG_NVFP4_SWIZZLED_SCALES:
                self.scales_fp4 = torch.empty(nvfp4_swizzled_scale_bytes(rows, H), dtype=u8,
                                              device=device)
                self.scales_mx4 = torch.empty(nvfp4_swizzled_scale_bytes(rows, H, 32),
                                              dtype=u8, device=device)
            else:
                self.scales_fp4 = torch.empty((max(rows, 1), max(H // 16, 1)), dtype=u8,
                                              device=device)
                self.scales_mx4 = torch.empty((max(rows, 1), max(H // 32, 1)), dtype=u8,
                                              device=device)
            self.out_mx4 = torch.empty((max(rows, 1), H // 2), dtype=u8, device=device)


def layout(prob: Problem, topk_ids: torch.Tensor, buf: Buffers, stream=None) -> None:
    moe_dispatch_layout(prob, topk_ids, buf.expert_counts, buf.expert_offsets, buf.meta,
                        buf.row_src, buf.pair_slot, buf.drop_mask, buf.status, buf.workspace,
                        stream)
