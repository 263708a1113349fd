"""The kernels' number conversions against the oracle, exhaustively.

The permutes and the SwiGLU quantiser turn fp32 values into E4M3 and E2M1
codes with the hardware conversions cvt.rn.satfinite.{e4m3x2,e2m1x2}.f32
(csrc/common.cuh: cvt_e4m3x4, cvt_e2m1x8), and divide by block scales with
rn_quotient2 (one correctly rounded reciprocal, two correction steps).  The
parity tests only reach the values bf16 data produces; here

  * every one of the 2^32 fp32 bit patterns goes through cvt_e4m3x4 and
    cvt_e2m1x8 and the codes are compared with the oracle's converters
    (written from the OCP format definitions).  NaN inputs: E4M3 must give
    a NaN code (either sign); E2M1 has no NaN and the contract excludes NaN
    inputs (the quotients the kernels convert are finite), so they are
    skipped;
  * rn_quotient2 is compared with IEEE fp32 division (numpy, on the CPU)
    over random and near-tie (a, d) pairs inside its guard: d in
    [2^-90, 2^124], |a / d| <= 2^24.  Quotients of magnitude at least 2^-13
    must be identical; smaller ones must be below 2^-12 in magnitude with
    the sign of a (every code here rounds them to the same signed zero).

The CUDA side is a test-only harness (tests/cuda/cvt_check.cu) built here
against the library's helper header; it is not part of libmoedc.so.
"""
import concurrent.futures as cf
import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "cuda", "cvt_check.cu")
LIB = os.path.join(HERE, "cuda", "libcvtcheck.so")
CHUNK = 1 << 26


@pytest.fixture(scope="module")
def harness():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from combine_topk_ids_scan_b200 import build
    deps = [SRC, os.path.join(ROOT, "combine_topk_ids_scan_b200", "csrc", "common.cuh")]
    if not os.path.exists(LIB) or os.path.getmtime(LIB) < max(map(os.path.getmtime, deps)):
        tmp = LIB + f".tmp{os.getpid()}"
        subprocess.run([build._nvcc(), *build.ARCH_FLAGS, "-O3", "-std=c++17", "-Xcompiler",
                        "-fPIC", "-shared", "-I", build.CSRC, "-I", build.INCLUDE, "-o", tmp,
                        SRC], check=True)
        os.replace(tmp, LIB)
    L = ctypes.CDLL(LIB)
    vp = ctypes.c_void_p
    for fn in ("cvt_check_e4m3", "cvt_check_e2m1"):
        getattr(L, fn).argtypes = [ctypes.c_uint32, ctypes.c_int64, vp, vp]
        getattr(L, fn).restype = ctypes.c_int
    L.cvt_check_quotient.argtypes = [vp, vp, vp, ctypes.c_int64, vp]
    L.cvt_check_quotient.restype = ctypes.c_int
    return L


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def _oracle_codes(fn, bits: np.ndarray) -> np.ndarray:
    """fn over bits.view(float32) in threads (single-threaded C per call)."""
    x = bits.view(np.float32)
    step = 1 << 21
    with cf.ThreadPoolExecutor(min(32, os.cpu_count() or 1)) as ex:
        parts = list(ex.map(lambda i: fn(x[i:i + step]), range(0, x.size, step)))
    return np.concatenate(parts)


def _is_nan(bits: np.ndarray) -> np.ndarray:
    return ((bits & 0x7F800000) == 0x7F800000) & ((bits & 0x007FFFFF) != 0)


@pytest.mark.parametrize("fmt", ["e4m3", "e2m1"])
def test_every_fp32_pattern_converts_like_the_oracle(orc, harness, fmt):
    call = harness.cvt_check_e4m3 if fmt == "e4m3" else harness.cvt_check_e2m1
    oracle_fn = orc.e4m3_from_f32 if fmt == "e4m3" else orc.e2m1_from_f32
    out = torch.empty(CHUNK, dtype=torch.uint8, device="cuda")
    checked = 0
    for c in range((1 << 32) // CHUNK):
        start = c * CHUNK
        assert call(start, CHUNK, ctypes.c_void_p(out.data_ptr()), _stream()) == 0
        got = out.cpu().numpy()
        bits = np.arange(start, start + CHUNK, dtype=np.uint64).astype(np.uint32)
        want = _oracle_codes(oracle_fn, bits)
        nan = _is_nan(bits)
        if fmt == "e4m3":
            assert np.all((got[nan] & 0x7F) == 0x7F), f"chunk {c}: NaN input, non-NaN code"
        ok = ~nan
        bad = np.flatnonzero(got[ok] != want[ok])
        assert bad.size == 0, (f"chunk {c}: {bad.size} mismatches, first pattern "
                               f"{int(bits[ok][bad[0]]):#010x}: gpu {int(got[ok][bad[0]]):#x} "
                               f"oracle {int(want[ok][bad[0]]):#x}")
        checked += int(ok.sum())
    assert checked == (1 << 32) - ((1 << 24) - 2)      # every pattern but the NaNs


def _quotient_pairs(rng, n):
    """n divisors d inside the guard and, for each, two numerators a (an
    [n, 2] array) with |a / d| <= 2^24: half of the quotients random, half
    on (or next to) the midpoint of two floats."""
    e = rng.integers(-90, 124, size=n)
    d = np.ldexp(rng.uniform(1.0, 2.0, size=n), e).astype(np.float32)
    d = np.clip(d, np.float32(2.0 ** -90), np.float32(2.0 ** 124))
    d[:4] = [2.0 ** -90, 2.0 ** 124, np.nextafter(np.float32(2.0 ** -90), np.float32(1)), 1.0]
    q = np.exp2(rng.uniform(-40.0, 23.9, size=(n, 2))) * np.where(rng.random((n, 2)) < 0.5,
                                                                  -1.0, 1.0)
    half = n // 2
    q32 = q[half:].astype(np.float32)
    ulp = np.spacing(np.abs(q32)).astype(np.float64)
    q[half:] = q32.astype(np.float64) + np.sign(q32) * ulp * rng.choice(
        [0.5, 0.5, 0.49, 0.51], size=q32.shape)
    a = np.clip(q * d.astype(np.float64)[:, None], -3.0e38, 3.0e38).astype(np.float32)
    return _within_guard(a, d), d


def _within_guard(a, d):
    """Halve (then zero) numerators whose quotient exceeds 2^24 after rounding."""
    for _ in range(2):
        over = np.abs(a.astype(np.float64) / d.astype(np.float64)[:, None]) > 2.0 ** 24
        a[over] = np.float32(0.5) * a[over]
    over = np.abs(a.astype(np.float64) / d.astype(np.float64)[:, None]) > 2.0 ** 24
    a[over] = np.float32(0.0)
    return a


@pytest.mark.parametrize("kind", ["fp32", "bf16"])
def test_rn_quotient_matches_ieee_division(harness, kind):
    rng = np.random.default_rng(77 if kind == "fp32" else 78)
    n = 1 << 23
    a2, d1 = _quotient_pairs(rng, n)
    if kind == "bf16":
        # the kernels divide bf16 data: round a to bf16 (nearest even)
        a2 = _within_guard(torch.from_numpy(a2).to(torch.bfloat16).to(torch.float32).numpy(), d1)
    a2 = np.ascontiguousarray(a2)
    a_dev = torch.from_numpy(a2).cuda()
    d_dev = torch.from_numpy(d1).cuda()
    q_dev = torch.empty_like(a_dev)
    assert harness.cvt_check_quotient(ctypes.c_void_p(a_dev.data_ptr()),
                                      ctypes.c_void_p(d_dev.data_ptr()),
                                      ctypes.c_void_p(q_dev.data_ptr()), n, _stream()) == 0
    got = q_dev.cpu().numpy()
    dd = np.repeat(d1[:, None], 2, axis=1)
    want = a2 / dd                                    # IEEE fp32 division, nearest even
    exact = np.abs(a2.astype(np.float64) / dd.astype(np.float64))
    big = exact >= 2.0 ** -13 * (1 + 2.0 ** -40)
    mism = np.flatnonzero((got != want) & big)
    assert mism.size == 0, (mism.size, float(a2.reshape(-1)[mism[0]]),
                            float(dd.reshape(-1)[mism[0]]))
    small = ~big
    assert np.all(np.abs(got[small]) < 2.0 ** -12)
    assert np.all(np.signbit(got[small]) == np.signbit(a2[small]))
    assert big.sum() > n          # most pairs take the exact branch
