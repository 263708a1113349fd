"""CPU oracle for MoE token dispatch and combine -- TEST INFRASTRUCTURE ONLY.

Only the test suite, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  The product path (the C-ABI library in
``combine_topk_ids_scan_b200``) never touches it, and the two share no code.

The arithmetic lives in ``oracle.c`` (plain single-threaded C, built with gcc
without fast-math or FP contraction).  This module only builds that file and
marshals numpy arrays to it.  Page citations for every function are in
``oracle.h`` / ``oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_HDR = os.path.join(_HERE, "oracle.h")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")

STATUS_ID_RANGE = 1
STATUS_DUP_ID = 2
STATUS_CAPACITY = 4
FLAG_CHECK_DUPLICATES = 1

_lib = None


def build(force: bool = False) -> str:
    """Compile oracle.c into liboracle.so next to it (gcc, -O2, IEEE)."""
    newest = max(os.path.getmtime(_SRC), os.path.getmtime(_HDR))
    if not force and os.path.exists(_LIB_PATH) and os.path.getmtime(_LIB_PATH) >= newest:
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-std=c11", "-O2", "-ffp-contract=off", "-fno-fast-math",
           "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


# Every output buffer handed to the C code is filled with a poison byte and
# followed by a guard of _GUARD poison bytes: an element the oracle fails to
# write keeps the poison (and fails the value checks), and a write past the
# end of the buffer is reported by _Outs.check.
_GUARD = 64
_POISON = 0xA5


class _Outs:
    """Allocator of poisoned, guarded output arrays for one oracle call."""

    def __init__(self):
        self._bufs = []

    def __call__(self, shape, dtype) -> np.ndarray:
        dt = np.dtype(dtype)
        shape = tuple(int(d) for d in np.atleast_1d(shape)) if np.ndim(shape) else (int(shape),)
        n = int(np.prod(shape, dtype=np.int64)) * dt.itemsize
        raw = np.full(n + _GUARD, _POISON, np.uint8)
        self._bufs.append((raw, n))
        return raw[:n].view(dt).reshape(shape)

    def check(self, fn: str) -> None:
        for raw, n in self._bufs:
            if not np.all(raw[n:] == _POISON):
                raise RuntimeError(f"{fn} wrote past the end of an output buffer")


def _p(a: np.ndarray | None):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(ctypes.c_void_p)


def lib():
    global _lib
    if _lib is None:
        L = ctypes.CDLL(build())
        i32, i64, u32, f32, vp = (ctypes.c_int32, ctypes.c_int64, ctypes.c_uint32,
                                  ctypes.c_float, ctypes.c_void_p)
        L.orc_layout.restype = u32
        L.orc_layout.argtypes = [i32, i32, i32, i32, i64, i32, i32, u32, i32,
                                 vp, vp, vp, vp, vp, vp, vp]
        L.orc_swizzle_scales.argtypes = [i64, i32, vp, vp]
        L.orc_permute_bf16.argtypes = [i64, i32, vp, vp, vp]
        L.orc_permute_fp8.argtypes = [i64, i32, vp, vp, vp, vp]
        L.orc_permute_nvfp4.argtypes = [i64, i32, vp, vp, f32, vp, vp]
        L.orc_permute_mxfp4.argtypes = [i64, i32, vp, vp, vp, vp]
        L.orc_pack_fp6.argtypes = [vp, i64, vp]
        L.orc_combine.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp]
        L.orc_permute_backward.argtypes = [i32, i32, i32, i64, vp, vp, vp]
        L.orc_permute_premultiplied.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp]
        L.orc_exp.restype = f32
        L.orc_exp.argtypes = [f32]
        L.orc_silu.restype = f32
        L.orc_silu.argtypes = [f32]
        L.orc_exp_n.argtypes = [vp, vp, i64]
        L.orc_e8m0_from_exponent.restype = ctypes.c_uint8
        L.orc_e8m0_from_exponent.argtypes = [i32]
        L.orc_swiglu_quant.argtypes = [i64, i32, vp, ctypes.c_int, vp, ctypes.c_int, f32, vp, vp]
        L.orc_combine_backward.argtypes = [i32, i32, i32, i64, vp, vp, vp, vp, vp, vp]
        for n in ("orc_bf16_from_f32_n", "orc_e4m3_from_f32_n", "orc_e2m1_from_f32_n",
                  "orc_e2m3_from_f32_n", "orc_e3m2_from_f32_n"):
            getattr(L, n).argtypes = [vp, vp, i64]
        for n in ("orc_e2m3_to_f32", "orc_e3m2_to_f32"):
            getattr(L, n).restype = f32
            getattr(L, n).argtypes = [ctypes.c_uint8]
        L.orc_e4m3_to_f32.restype = f32
        L.orc_e4m3_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_e2m1_to_f32.restype = f32
        L.orc_e2m1_to_f32.argtypes = [ctypes.c_uint8]
        L.orc_bf16_to_f32.restype = f32
        L.orc_bf16_to_f32.argtypes = [ctypes.c_uint16]
        _lib = L
    return _lib


# ---------------------------------------------------------------- formats
def bf16_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.uint16)
    lib().orc_bf16_from_f32_n(_p(x), _p(out), x.size)
    o.check("orc_bf16_from_f32_n")
    return out


def e4m3_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.uint8)
    lib().orc_e4m3_from_f32_n(_p(x), _p(out), x.size)
    o.check("orc_e4m3_from_f32_n")
    return out


def e2m1_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.uint8)
    lib().orc_e2m1_from_f32_n(_p(x), _p(out), x.size)
    o.check("orc_e2m1_from_f32_n")
    return out


def e2m3_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.uint8)
    lib().orc_e2m3_from_f32_n(_p(x), _p(out), x.size)
    o.check("orc_e2m3_from_f32_n")
    return out


def e3m2_from_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.uint8)
    lib().orc_e3m2_from_f32_n(_p(x), _p(out), x.size)
    o.check("orc_e3m2_from_f32_n")
    return out


def e2m3_to_f32(code: int) -> float:
    return float(lib().orc_e2m3_to_f32(code))


def e3m2_to_f32(code: int) -> float:
    return float(lib().orc_e3m2_to_f32(code))


def pack_fp6(codes: np.ndarray) -> np.ndarray:
    codes = np.ascontiguousarray(codes, dtype=np.uint8).reshape(-1)
    o = _Outs()
    out = o(codes.size * 3 // 4, np.uint8)
    lib().orc_pack_fp6(_p(codes), codes.size, _p(out))
    o.check("orc_pack_fp6")
    return out


def e4m3_to_f32(code: int) -> float:
    return lib().orc_e4m3_to_f32(code)


def e2m1_to_f32(code: int) -> float:
    return lib().orc_e2m1_to_f32(code)


# ---------------------------------------------------------------- layout
class Layout:
    """Outputs of the dispatch layout for one problem."""

    def __init__(self, status, expert_counts, expert_offsets, meta, row_src,
                 pair_slot, drop_mask):
        self.status = status
        self.expert_counts = expert_counts
        self.expert_offsets = expert_offsets
        self.meta = meta
        self.row_src = row_src
        self.pair_slot = pair_slot
        self.drop_mask = drop_mask


def layout(ids: np.ndarray, num_experts: int, num_segments: int, hidden: int,
           recv_capacity: int = 0, expert_capacity: int = 0,
           flags: int = 0, expert_pad_multiple: int = 0) -> Layout:
    ids = np.ascontiguousarray(ids, dtype=np.int32)
    N, k = ids.shape
    E, S = num_experts, num_segments
    rows = E * expert_capacity if expert_capacity > 0 else recv_capacity
    o = _Outs()
    counts = o(E, np.int32)
    offsets = o(E + 1, np.int32)
    meta = o((4, S), np.uint32)
    row_src = o(rows, np.int32)
    pair_slot = o((N, k), np.int32)
    drop = o((N, k), np.uint8)
    st = lib().orc_layout(N, k, E, S, recv_capacity, expert_capacity, expert_pad_multiple,
                          flags, hidden,
                          _p(ids), _p(counts), _p(offsets), _p(meta), _p(row_src),
                          _p(pair_slot), _p(drop))
    o.check("orc_layout")
    return Layout(int(st), counts, offsets, meta, row_src, pair_slot, drop)


# ---------------------------------------------------------------- permute
def permute_bf16(hidden_bits: np.ndarray, row_src: np.ndarray) -> np.ndarray:
    """hidden_bits: uint16 [N,H] bf16 bit patterns; returns uint16 [rows,H]."""
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    row_src = np.ascontiguousarray(row_src, dtype=np.int32)
    H = hidden_bits.shape[1]
    o = _Outs()
    out = o((row_src.size, H), np.uint16)
    lib().orc_permute_bf16(row_src.size, H, _p(hidden_bits), _p(row_src), _p(out))
    o.check("orc_permute_bf16")
    return out


def permute_fp8(hidden_bits: np.ndarray, row_src: np.ndarray):
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    row_src = np.ascontiguousarray(row_src, dtype=np.int32)
    H = hidden_bits.shape[1]
    o = _Outs()
    q = o((row_src.size, H), np.uint8)
    sc = o((row_src.size, H // 128), np.float32)
    lib().orc_permute_fp8(row_src.size, H, _p(hidden_bits), _p(row_src), _p(q), _p(sc))
    o.check("orc_permute_fp8")
    return q, sc


def permute_nvfp4(hidden_bits: np.ndarray, row_src: np.ndarray, global_scale: float):
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    row_src = np.ascontiguousarray(row_src, dtype=np.int32)
    H = hidden_bits.shape[1]
    o = _Outs()
    q = o((row_src.size, H // 2), np.uint8)
    sc = o((row_src.size, H // 16), np.uint8)
    lib().orc_permute_nvfp4(row_src.size, H, _p(hidden_bits), _p(row_src),
                            float(np.float32(global_scale)), _p(q), _p(sc))
    o.check("orc_permute_nvfp4")
    return q, sc


def permute_mxfp4(hidden_bits: np.ndarray, row_src: np.ndarray):
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    row_src = np.ascontiguousarray(row_src, dtype=np.int32)
    H = hidden_bits.shape[1]
    o = _Outs()
    q = o((row_src.size, H // 2), np.uint8)
    sc = o((row_src.size, H // 32), np.uint8)
    lib().orc_permute_mxfp4(row_src.size, H, _p(hidden_bits), _p(row_src), _p(q), _p(sc))
    o.check("orc_permute_mxfp4")
    return q, sc


def swizzle_scales(linear: np.ndarray) -> np.ndarray:
    """[rows, nsf] uint8 scales -> the 128x4 atom layout (flat uint8)."""
    linear = np.ascontiguousarray(linear, dtype=np.uint8)
    rows, nsf = linear.shape
    o = _Outs()
    out = o(((rows + 127) // 128 * 128) * ((nsf + 3) // 4 * 4), np.uint8)
    lib().orc_swizzle_scales(rows, nsf, _p(linear), _p(out))
    o.check("orc_swizzle_scales")
    return out


# ---------------------------------------------------------------- combine
def combine(expert_out_bits: np.ndarray, gates: np.ndarray,
            pair_slot: np.ndarray) -> np.ndarray:
    """expert_out_bits: uint16 [rows,H] bf16; gates f32 [N,k]; returns uint16 [N,H]."""
    expert_out_bits = np.ascontiguousarray(expert_out_bits, dtype=np.uint16)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    pair_slot = np.ascontiguousarray(pair_slot, dtype=np.int32)
    N, k = pair_slot.shape
    rows, H = expert_out_bits.shape
    o = _Outs()
    y = o((N, H), np.uint16)
    lib().orc_combine(N, k, H, rows, _p(expert_out_bits), _p(gates), _p(pair_slot), _p(y))
    o.check("orc_combine")
    return y


# ---------------------------------------------------------------- backward
def permute_backward(grad_out_bits: np.ndarray, pair_slot: np.ndarray) -> np.ndarray:
    """grad_out: uint16 [rows,H] bf16; returns grad_hidden uint16 [N,H]."""
    grad_out_bits = np.ascontiguousarray(grad_out_bits, dtype=np.uint16)
    pair_slot = np.ascontiguousarray(pair_slot, dtype=np.int32)
    N, k = pair_slot.shape
    rows, H = grad_out_bits.shape
    o = _Outs()
    gh = o((N, H), np.uint16)
    lib().orc_permute_backward(N, k, H, rows, _p(grad_out_bits), _p(pair_slot), _p(gh))
    o.check("orc_permute_backward")
    return gh


def combine_backward(grad_y_bits: np.ndarray, expert_out_bits: np.ndarray, gates: np.ndarray,
                     pair_slot: np.ndarray):
    """Returns (grad_expert_out uint16 [rows,H], grad_gates float32 [N,k])."""
    grad_y_bits = np.ascontiguousarray(grad_y_bits, dtype=np.uint16)
    expert_out_bits = np.ascontiguousarray(expert_out_bits, dtype=np.uint16)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    pair_slot = np.ascontiguousarray(pair_slot, dtype=np.int32)
    N, k = pair_slot.shape
    rows, H = expert_out_bits.shape
    o = _Outs()
    gx = o((rows, H), np.uint16)
    gw = o((N, k), np.float32)
    lib().orc_combine_backward(N, k, H, rows, _p(grad_y_bits), _p(expert_out_bits), _p(gates),
                               _p(pair_slot), _p(gx), _p(gw))
    o.check("orc_combine_backward")
    return gx, gw


# ---------------------------------------------------------------- pre-multiplied gates
def permute_premultiplied(hidden_bits: np.ndarray, gates: np.ndarray, pair_slot: np.ndarray,
                          rows: int) -> np.ndarray:
    """hidden: uint16 [N,H] bf16; gates f32 [N,k]; returns uint16 [rows,H]:
    each pair's row is its token scaled by its gate (zeros elsewhere)."""
    hidden_bits = np.ascontiguousarray(hidden_bits, dtype=np.uint16)
    gates = np.ascontiguousarray(gates, dtype=np.float32)
    pair_slot = np.ascontiguousarray(pair_slot, dtype=np.int32)
    N, k = pair_slot.shape
    H = hidden_bits.shape[1]
    o = _Outs()
    out = o((rows, H), np.uint16)
    lib().orc_permute_premultiplied(N, k, H, rows, _p(hidden_bits), _p(gates), _p(pair_slot),
                                    _p(out))
    o.check("orc_permute_premultiplied")
    return out


# ---------------------------------------------------------------- SwiGLU
FMT_NVFP4, FMT_MXFP8, FMT_MXFP4, FMT_BF16, FMT_MXFP6_E2M3, FMT_MXFP6_E3M2 = 0, 1, 2, 3, 4, 5


def swiglu_code_bytes(I: int, fmt: int) -> int:
    """Bytes of one row of swiglu_quant codes."""
    return {FMT_NVFP4: I // 2, FMT_MXFP8: I, FMT_MXFP4: I // 2, FMT_BF16: 2 * I,
            FMT_MXFP6_E2M3: 3 * I // 4, FMT_MXFP6_E3M2: 3 * I // 4}[fmt]


def swiglu_scale_bytes(I: int, fmt: int) -> int:
    """Bytes of one row of swiglu_quant scales (0 for bf16)."""
    return I // 16 if fmt == FMT_NVFP4 else 0 if fmt == FMT_BF16 else I // 32


def exp_f32(x: np.ndarray) -> np.ndarray:
    x = np.ascontiguousarray(x, dtype=np.float32)
    o = _Outs()
    out = o(x.shape, np.float32)
    lib().orc_exp_n(_p(x), _p(out), x.size)
    o.check("orc_exp_n")
    return out


def swiglu_quant(gate_up_bits: np.ndarray, row_src: np.ndarray, fmt: int,
                 interleaved: bool = False, global_scale: float = 1.0):
    """gate_up: uint16 [rows, 2I] bf16 bits; returns (codes, scales) uint8."""
    gate_up_bits = np.ascontiguousarray(gate_up_bits, dtype=np.uint16)
    row_src = np.ascontiguousarray(row_src, dtype=np.int32)
    rows, two_i = gate_up_bits.shape
    I = two_i // 2
    o = _Outs()
    codes = o((rows, swiglu_code_bytes(I, fmt)), np.uint8)
    scales = o((rows, swiglu_scale_bytes(I, fmt)), np.uint8)
    lib().orc_swiglu_quant(rows, I, _p(gate_up_bits), int(interleaved), _p(row_src), fmt,
                           float(np.float32(global_scale)), _p(codes), _p(scales))
    o.check("orc_swiglu_quant")
    return codes, scales
