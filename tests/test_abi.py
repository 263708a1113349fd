"""CPU-side checks of the C ABI: the library builds for sm_100a, loads,
exports every entry point include/moe_dc.h declares, and its host-side logic
(sizes, workspace, argument validation) behaves -- without launching anything."""
import ctypes
import os
import re
import subprocess

import pytest

from combine_topk_ids_scan_b200 import binding as B
from combine_topk_ids_scan_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def lib():
    build.build()
    return B.load()


def declared_functions():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            names |= set(re.findall(r"\b(moe_\w+)\s*\(", src))
    return names


def test_every_declared_symbol_is_exported(lib):
    declared = declared_functions()
    assert declared == set(B.EXPORTED)
    out = subprocess.run(["nm", "-D", "--defined-only", B.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = set(re.findall(r"\bT (moe_\w+)", out))
    assert declared <= exported, declared - exported
    # nothing else leaks out under the moe_ prefix
    assert exported == declared


def test_built_for_sm100a(lib):
    out = subprocess.run(["cuobjdump", "--list-elf", B.LIB_PATH], capture_output=True,
                         text=True)
    if out.returncode == 0:
        assert "sm_100a" in out.stdout


def test_host_only_entry_points(lib):
    assert B.version().startswith("moedc")
    assert B.debug_violations() == -1          # the normal build has no device checks
    assert "invalid" in B.status_string(B.MOE_ERR_INVALID_ARG)
    p = B.Problem(num_tokens=8192, hidden=7168, num_experts=256, top_k=8, num_segments=8,
                  recv_capacity=65536)
    assert B.moe_output_rows(p) == 65536
    # control (256 B) + totals (1 KiB) + 16 scan tiles x 256 experts x 8 B
    assert B.moe_workspace_bytes(p) == 256 + 1024 + 16 * 256 * 8
    p.expert_capacity = 5
    assert B.moe_output_rows(p) == 1280
    p.num_segments = 3
    assert B.moe_output_rows(p) == -1 and B.moe_workspace_bytes(p) == 0


def _call(lib, fn, prob, nptr):
    c = prob.c()
    return getattr(lib, fn)(ctypes.byref(c), *([None] * nptr))


@pytest.mark.parametrize("mutate,code", [
    (dict(num_segments=3), B.MOE_ERR_UNSUPPORTED_SHAPE),        # E % S != 0
    (dict(num_experts=4096, num_segments=1), B.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(top_k=17), B.MOE_ERR_UNSUPPORTED_SHAPE),
    (dict(num_tokens=-1), B.MOE_ERR_INVALID_ARG),
    (dict(hidden=0), B.MOE_ERR_INVALID_ARG),
    (dict(recv_capacity=1 << 40), B.MOE_ERR_UNSUPPORTED_SHAPE),  # int32 rows
    (dict(hidden=1 << 20, recv_capacity=1 << 13), B.MOE_ERR_UNSUPPORTED_SHAPE),  # uint32 meta
    ({}, B.MOE_ERR_INVALID_ARG),                                  # null pointers
])
def test_layout_validation(lib, mutate, code):
    p = B.Problem(num_tokens=100, hidden=64, num_experts=8, top_k=2, num_segments=2,
                  recv_capacity=200)
    for k, v in mutate.items():
        setattr(p, k, v)
    assert _call(lib, "moe_dispatch_layout", p, 10) == code


def test_payload_shape_rules(lib):
    p = B.Problem(num_tokens=10, hidden=100, num_experts=8, top_k=2, num_segments=2,
                  recv_capacity=20)
    assert _call(lib, "moe_permute", p, 5) == B.MOE_ERR_UNSUPPORTED_SHAPE       # H % 8
    assert _call(lib, "moe_combine", p, 5) == B.MOE_ERR_UNSUPPORTED_SHAPE
    assert _call(lib, "moe_permute_premultiplied", p, 6) == B.MOE_ERR_UNSUPPORTED_SHAPE
    p.hidden = 96
    assert _call(lib, "moe_permute_quant_fp8", p, 6) == B.MOE_ERR_UNSUPPORTED_SHAPE  # H % 128
    p.hidden = 80
    assert _call(lib, "moe_permute_quant_nvfp4", p, 7) == B.MOE_ERR_UNSUPPORTED_SHAPE  # H % 32
    p.hidden = 128
    for fn, n in (("moe_permute", 5), ("moe_permute_premultiplied", 6),
                  ("moe_permute_quant_fp8", 6),
                  ("moe_permute_quant_nvfp4", 7), ("moe_combine", 5)):
        assert _call(lib, fn, p, n) == B.MOE_ERR_INVALID_ARG, fn      # null pointers
    assert lib.moe_permute(None, *([None] * 5)) == B.MOE_ERR_INVALID_ARG
    bad = B.moe_problem(10, 128, 8, 2, 2, 0, 20, 0, -3)                  # negative pad
    assert lib.moe_combine(ctypes.byref(bad), *([None] * 5)) == B.MOE_ERR_INVALID_ARG
    bad = B.moe_problem(10, 128, 8, 2, 2, 4, 0, 0, 8)                    # pad with Ce
    assert lib.moe_combine(ctypes.byref(bad), *([None] * 5)) == B.MOE_ERR_INVALID_ARG


def test_next_row_argument_rules(lib):
    """MX dispatch, SwiGLU and backward entry points reject bad shapes and
    arguments on the host, before anything is launched."""
    p = B.Problem(num_tokens=10, hidden=80, num_experts=8, top_k=2, num_segments=2,
                  recv_capacity=20)
    assert _call(lib, "moe_permute_quant_mxfp4", p, 6) == B.MOE_ERR_UNSUPPORTED_SHAPE  # H % 32
    p.hidden = 128
    assert _call(lib, "moe_permute_quant_mxfp4", p, 6) == B.MOE_ERR_INVALID_ARG        # nulls
    assert _call(lib, "moe_permute_backward", p, 4) == B.MOE_ERR_INVALID_ARG
    assert _call(lib, "moe_combine_backward", p, 8) == B.MOE_ERR_INVALID_ARG
    c = p.c()
    sw = lib.moe_swiglu_quant
    vp = [None] * 6
    assert sw(ctypes.byref(c), 96, 6, 0, *vp) == B.MOE_ERR_INVALID_ARG          # format
    assert sw(ctypes.byref(c), 96, 1, 2, *vp) == B.MOE_ERR_INVALID_ARG          # gate/up layout
    assert sw(ctypes.byref(c), 0, 1, 0, *vp) == B.MOE_ERR_INVALID_ARG           # I <= 0
    assert sw(ctypes.byref(c), 100, 1, 0, *vp) == B.MOE_ERR_UNSUPPORTED_SHAPE   # I % 32
    for fmt in range(6):
        assert sw(ctypes.byref(c), 96, fmt, 0, *vp) == B.MOE_ERR_INVALID_ARG    # null pointers
    # misaligned codes (MXFP6 needs 8 bytes, the others 16): reported, nothing launched
    buf = ctypes.create_string_buffer(4096)
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    ptrs = [base, base + 256, base + 512, base + 1024 + 8, base + 2048]  # gate_up, row_src, gs, codes, scales
    assert sw(ctypes.byref(c), 96, 1, 0, ptrs[0], ptrs[1], ptrs[2], ptrs[3], ptrs[4],
              None) == B.MOE_ERR_INVALID_ARG


# entry point -> (fixed leading arguments after the problem, the pointer
# arguments' required alignment in bytes (1: none); a trailing stream of None)
ALIGNMENT_RULES = {
    "moe_dispatch_layout": ((), (4, 4, 4, 4, 4, 4, 1, 4, 16)),
    "moe_dispatch_layout_noalloc": ((), (4, 4, 4, 4, 4, 4, 1, 4)),
    "moe_permute": ((), (16, 4, 4, 16)),
    "moe_permute_premultiplied": ((), (16, 4, 4, 4, 16)),
    "moe_permute_to_peers": ((), (16, 4, 4, 4, 8, 8)),
    "moe_permute_quant_fp8_to_peers": ((), (16, 4, 4, 4, 8, 8, 8)),
    "moe_permute_quant_nvfp4_to_peers": ((), (16, 4, 4, 4, 4, 8, 8, 8)),
    "moe_permute_quant_fp8": ((), (16, 4, 4, 16, 4)),
    "moe_permute_quant_nvfp4": ((), (16, 4, 4, 4, 16, 2)),
    "moe_permute_quant_mxfp4": ((), (16, 4, 4, 16, 1)),
    "moe_combine": ((), (16, 4, 4, 16)),
    "moe_combine_from_peers": ((), (8, 8, 4, 4, 4, 16)),
    "moe_permute_backward": ((), (16, 4, 16)),
    "moe_combine_backward": ((), (16, 16, 4, 4, 4, 16, 4)),
    "moe_swiglu_quant": ((128, 0, 0), (16, 4, 4, 16, 2)),   # I = 128, NVFP4, split
}


def test_every_pointer_alignment_is_checked_on_the_host(lib):
    """Each call gets aligned, non-null (host) addresses except for one
    misaligned pointer, and must reject it before launching anything.
    Skipped where a GPU is present: the addresses are not device memory."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("host-side argument checks only; run on a machine without a GPU")
    buf = ctypes.create_string_buffer(64 * 256 + 256)
    base = (ctypes.addressof(buf) + 255) // 256 * 256
    p = B.Problem(num_tokens=10, hidden=128, num_experts=8, top_k=2, num_segments=2,
                  recv_capacity=20)
    c = p.c()
    checked = 0
    for fn, (lead, aligns) in ALIGNMENT_RULES.items():
        for i, a in enumerate(aligns):
            for off in sorted({a // 2, 1} - {0}) if a > 1 else []:
                ptrs = [base + 256 * n for n in range(len(aligns))]
                ptrs[i] += off
                rc = getattr(lib, fn)(ctypes.byref(c), *lead, *ptrs, None)
                assert rc == B.MOE_ERR_INVALID_ARG, (fn, i, a, off, rc)
                checked += 1
    assert checked > 60


def test_missing_library_fails_loudly(tmp_path, monkeypatch):
    monkeypatch.setattr(B, "_lib", None)
    with pytest.raises(RuntimeError, match="not found"):
        B.load(str(tmp_path / "nope.so"))
