"""Pins for the oracle's MX token format (MXFP4 dispatch), its OCP MX FP6
element codecs (E2M3, E3M2), the packed 6-bit layout, and the SwiGLU bf16 /
MXFP6 outputs (CPU only).

The FP6 value tables come from the OCP Microscaling v1.0 specification
(tests/golden/fp6_values.txt); encoders are checked against an arithmetic
round-to-nearest-even written here (scaled significand, Python's
round-half-even), which is a different method from the oracle's search over
the code table; MX blocks against the shared-scale rule worked out here with
math.frexp; bf16 outputs against torch's bfloat16 cast.
"""
import math
import os

import numpy as np
import pytest
import torch

from test_oracle_swiglu import bf16_bits, f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "fp6_values.txt")
FMT = {"e2m3": (2, 3, 1, 7.5), "e3m2": (3, 2, 3, 28.0)}   # ebits, mbits, bias, max


def spec_table():
    rows = [l.split() for l in open(GOLDEN) if l.strip() and not l.startswith("#")]
    return {"e2m3": np.array([float(r[1]) for r in rows]),
            "e3m2": np.array([float(r[2]) for r in rows])}


def rne_fp6(x, fmt):
    """Round to nearest even on the FP6 grid by arithmetic: the grid step in
    a's binade is 2^(e - mbits) (the subnormal step below the smallest
    normal), a / step rounded half-to-even, saturating at the maximum."""
    ebits, mbits, bias, vmax = FMT[fmt]
    out = []
    for v in np.asarray(x, np.float64):
        a = abs(v)
        e = max(math.frexp(a)[1] - 1, 1 - bias) if a > 0 else 1 - bias
        step = 2.0 ** (e - mbits)
        q = vmax if a > 2 * vmax else min(round(a / step) * step, vmax)
        out.append(math.copysign(q, v))
    return np.array(out)


def decode(fmt, codes, orc):
    f = orc.e2m3_to_f32 if fmt == "e2m3" else orc.e3m2_to_f32
    return np.array([f(int(c)) for c in np.asarray(codes).reshape(-1)])


@pytest.mark.parametrize("fmt", ["e2m3", "e3m2"])
def test_fp6_decode_matches_spec_table(orc, fmt):
    tab = spec_table()[fmt]
    assert np.array_equal(decode(fmt, np.arange(32), orc), tab)
    neg = decode(fmt, np.arange(32, 64), orc)
    assert np.array_equal(neg, -tab) and math.copysign(1, neg[0]) < 0
    assert np.all(np.diff(tab) > 0)


@pytest.mark.parametrize("fmt", ["e2m3", "e3m2"])
def test_fp6_encode_round_nearest_even(orc, fmt):
    tab = spec_table()[fmt]
    enc = orc.e2m3_from_f32 if fmt == "e2m3" else orc.e3m2_from_f32
    rng = np.random.default_rng(11)
    mids = (tab[1:] + tab[:-1]) / 2
    x = np.concatenate([
        rng.uniform(-40, 40, 20000), rng.standard_normal(20000) * 0.3,
        mids, -mids, np.nextafter(mids, 0), np.nextafter(mids, 100),
        tab, -tab, [0.0, -0.0, 1e-30, -1e-30, 1e30, -1e30, np.inf, -np.inf]]).astype(np.float32)
    codes = enc(x)
    assert codes.max() < 64
    got = decode(fmt, codes, orc)
    want = rne_fp6(x, fmt)
    assert np.array_equal(got, want)
    # signs are kept, also for results of zero
    assert np.array_equal(codes >= 32, np.signbit(x))
    # every midpoint goes to the neighbour with the even code
    mc = enc(mids.astype(np.float32))
    assert np.all(mc % 2 == 0)


def test_pack_fp6_hand_example(orc):
    # codes 1, 2, 3, 4 -> 1 | 2<<6 | 3<<12 | 4<<18 = 0x103081, little-endian
    assert list(orc.pack_fp6(np.array([1, 2, 3, 4], np.uint8))) == [0x81, 0x30, 0x10]
    assert list(orc.pack_fp6(np.array([63, 0, 0, 0], np.uint8))) == [0x3F, 0, 0]
    assert list(orc.pack_fp6(np.array([0, 0, 0, 63], np.uint8))) == [0, 0, 0xFC]
    rng = np.random.default_rng(12)
    c = rng.integers(0, 64, 4000).astype(np.uint8)
    b = orc.pack_fp6(c).astype(np.uint32)
    w = b[0::3] | (b[1::3] << 8) | (b[2::3] << 16)
    back = np.stack([(w >> (6 * i)) & 0x3F for i in range(4)], axis=1).reshape(-1)
    assert np.array_equal(back, c)


def swiglu_y(orc, gu, I):
    gf, uf = f32(gu[:, :I]), f32(gu[:, I:])
    return np.array([[orc.lib().orc_silu(float(a)) for a in r] for r in gf], np.float32) * uf


def test_swiglu_bf16_output(orc):
    rng = np.random.default_rng(13)
    rows, I = 12, 96
    gu = bf16_bits(rng.standard_normal((rows, 2 * I)) * 3)
    src = np.arange(rows, dtype=np.int32)
    src[4] = -1
    codes, scales = orc.swiglu_quant(gu, src, orc.FMT_BF16)
    assert scales.shape == (rows, 0)
    y = swiglu_y(orc, gu, I)
    want = torch.from_numpy(y).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint8)
    want = want.reshape(rows, 2 * I).copy()
    want[4] = 0
    assert np.array_equal(codes, want)


@pytest.mark.parametrize("fmt", ["e2m3", "e3m2"])
def test_swiglu_mxfp6_block_rule(orc, fmt):
    """Per block: X = floor(log2(amax)) - emax (2 for E2M3, 4 for E3M2 --
    the exponent of the largest normal), scale code X + 127, codes the FP6
    RNE of y * 2^-X packed four to three bytes; all-zero block: scale 0."""
    rng = np.random.default_rng(14 + len(fmt))
    rows, I = 16, 128
    gu = bf16_bits(rng.standard_normal((rows, 2 * I)) * 2)
    gu[2, I:I + 32] = 0                       # an all-zero block (u = 0)
    gu[3, 32], gu[3, I + 32] = bf16_bits([8.0, 16.0])   # block max at its element 0
    gu[5, I + 64:I + 96] = bf16_bits(np.full(32, 1e-39))  # tiny block: the scale clamps
    src = np.arange(rows, dtype=np.int32)
    src[7] = -1
    f = orc.FMT_MXFP6_E2M3 if fmt == "e2m3" else orc.FMT_MXFP6_E3M2
    codes, scales = orc.swiglu_quant(gu, src, f)
    assert codes.shape == (rows, 3 * I // 4) and scales.shape == (rows, I // 32)
    y = swiglu_y(orc, gu, I)
    emax = 2 if fmt == "e2m3" else 4
    tab = spec_table()[fmt]
    for r in range(rows):
        if src[r] < 0:
            assert not codes[r].any() and not scales[r].any()
            continue
        b = codes[r].astype(np.uint32)
        w = b[0::3] | (b[1::3] << 8) | (b[2::3] << 16)
        c6 = np.stack([(w >> (6 * i)) & 0x3F for i in range(4)], axis=1).reshape(-1)
        for k in range(I // 32):
            blk = y[r, 32 * k:32 * k + 32].astype(np.float64)
            amax = np.abs(blk).max()
            if amax == 0:
                assert scales[r, k] == 0 and not c6[32 * k:32 * k + 32].any()
                continue
            # E8M0 holds 2^-127 .. 2^127: a smaller X takes the smallest scale
            X = max(math.frexp(amax)[1] - 1 - emax, -127)
            assert scales[r, k] == X + 127
            v = rne_fp6(blk * 2.0 ** -X, fmt)
            got = np.where(c6[32 * k:32 * k + 32] >= 32, -1.0, 1.0) * tab[c6[32 * k:32 * k + 32] & 31]
            assert np.array_equal(got, v)
            if X > -127:
                # the scaled block maximum lands in the top binade [2^emax, 2^(emax+1))
                assert 2.0 ** emax <= amax * 2.0 ** -X < 2.0 ** (emax + 1)
    blk = y[3, 32:64]
    assert np.argmax(np.abs(blk)) == 0 and np.abs(blk[0]) >= 2 * np.abs(blk[1:]).max()
    assert scales[5, 2] == 0 and 0 < np.abs(y[5, 64:96]).max() < 2.0 ** (-126 + emax)


def test_permute_mxfp4_block_rule(orc):
    """MX token format: per 32-element block of the bf16 row, X =
    floor(log2(amax)) - 2, E8M0 code X + 127, E2M1 RNE of x * 2^-X (element
    2m in the low nibble); zero blocks and padding rows all zero."""
    from test_oracle_formats import E2M1
    rng = np.random.default_rng(15)
    N, H = 20, 256
    x = bf16_bits(rng.standard_normal((N, H)) * np.exp(rng.uniform(-8, 8, (N, 1))))
    x[3, 32:64] = 0
    x[5, :32] = bf16_bits(np.full(32, -0.0, np.float32))
    x[9, :64] = rng.integers(1, 0x7F, 64).astype(np.uint16)        # bf16 subnormals
    x[9, 64:96] = 0x7F7F                                            # bf16 maximum
    x[7, 96:128] = bf16_bits(np.linspace(0.1, 0.2, 32))
    x[7, 96] = bf16_bits([-3.0])[0]                                 # block max at element 0
    row_src = np.array([0, 3, -1, 5, 19, 7, 3, -1, 9], np.int32)
    q, s = orc.permute_mxfp4(x, row_src)
    assert q.shape == (9, H // 2) and s.shape == (9, H // 32)
    val = {c: v for c, v in E2M1}
    for r, t in enumerate(row_src):
        if t < 0:
            assert not q[r].any() and not s[r].any()
            continue
        xf = f32(x[t]).astype(np.float64)
        codes = np.stack([q[r] & 0xF, q[r] >> 4], axis=1).reshape(-1)
        for k in range(H // 32):
            blk = xf[32 * k:32 * k + 32]
            amax = np.abs(blk).max()
            if amax == 0:
                assert s[r, k] == 0 and not codes[32 * k:32 * k + 32].any()
                continue
            X = min(max(math.frexp(amax)[1] - 1 - 2, -127), 127)   # E8M0 range
            assert s[r, k] == X + 127
            scaled = blk * 2.0 ** -X
            cc = codes[32 * k:32 * k + 32]
            got = np.where(cc >= 8, -1.0, 1.0) * np.array([val[c & 7] for c in cc])
            # E2M1 grid: step 0.5 below 2, 1 in [2, 4), 2 in [4, 6]
            a = np.abs(scaled)
            step = np.where(a < 2, 0.5, np.where(a < 4, 1.0, 2.0))
            want = np.minimum(np.array([round(v) for v in a / step]) * step, 6.0)
            assert np.array_equal(np.abs(got), want)
            assert np.array_equal(cc >= 8, np.signbit(scaled))
