"""Pins for the oracle's SwiGLU and its MX / NVFP4 requantisation (CPU only).

exp is checked against float64 math within 2 ulps; silu against its closed
forms; the MX shared-scale rule of the OCP Microscaling v1.0 specification
(X = floor(log2(amax)) - emax of the element format, E8M0 code X + 127) by
hand-computed blocks; element codes by brute-force nearest-even search; the
interleaved layout against the split one.
"""
import math

import numpy as np
import pytest
import torch

from test_oracle_formats import E2M1, brute_nearest_even, e4m3_table


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def ulps(a, b):
    a = np.asarray(a, np.float32).view(np.int32).astype(np.int64)
    b = np.asarray(b, np.float32).view(np.int32).astype(np.int64)
    return np.abs(a - b)


def test_exp_within_two_ulps(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([rng.uniform(-87, 88, 200000), rng.uniform(-1, 1, 50000),
                        [0.0, 1.0, -1.0, 88.0, -87.0]]).astype(np.float32)
    got = orc.exp_f32(x)
    want = np.exp(x.astype(np.float64)).astype(np.float32)
    assert np.all(ulps(got, want) <= 2)
    assert orc.exp_f32(np.array([0.0], np.float32))[0] == 1.0
    assert orc.exp_f32(np.array([100.0], np.float32))[0] == np.inf
    assert orc.exp_f32(np.array([-200.0], np.float32))[0] == 0.0


def test_exp_overflow_and_subnormal_tails(orc):
    """Near the ends of the float range: x in [88.38, 88.72] (n = 128, the
    result scaled in two steps) within 2 ulps of float64 exp, and inf once
    e^x is clearly past the largest float; x in [-103.9, -87.4] (subnormal
    results, scaled in two steps) within 2 ulps of the float64 value rounded
    to float32."""
    rng = np.random.default_rng(6)
    hi = np.concatenate([rng.uniform(88.38, 88.7228, 20000), [88.4, 88.5, 88.7]]).astype(np.float32)
    got = orc.exp_f32(hi)
    want = np.exp(hi.astype(np.float64))
    assert np.all(want < np.finfo(np.float32).max)
    assert np.all(ulps(got, want.astype(np.float32)) <= 2)
    over = np.array([88.7230, 88.73, 88.749], np.float32)
    assert np.all(np.exp(over.astype(np.float64)) > 1.0001 * float(np.finfo(np.float32).max))
    assert np.all(orc.exp_f32(over) == np.inf)
    lo = np.concatenate([rng.uniform(-103.9, -87.4, 20000), [-88.0, -100.0]]).astype(np.float32)
    got = orc.exp_f32(lo)
    want = np.exp(lo.astype(np.float64)).astype(np.float32)
    assert np.all(want < np.finfo(np.float32).tiny) and np.all(want > 0)
    assert np.all(ulps(got, want) <= 2)


def test_silu_closed_forms(orc):
    L = orc.lib()
    assert L.orc_silu(0.0) == 0.0
    for g in (30.0, 50.0, 88.0):              # e^-g below half an ulp of 1
        assert L.orc_silu(g) == g
    assert L.orc_silu(-200.0) == 0.0 and math.copysign(1, L.orc_silu(-200.0)) < 0
    rng = np.random.default_rng(2)
    for g in rng.uniform(-20, 20, 2000).astype(np.float32):
        want = float(g) / (1.0 + math.exp(-float(g)))
        assert ulps(L.orc_silu(float(g)), want) <= 3


@pytest.mark.parametrize("amax,fmt,code", [
    (6.0, 1, 121), (448.0, 1, 127), (1.0, 1, 119), (0.75, 1, 118), (1e-30, 1, 19),
    (6.0, 2, 127), (1.0, 2, 125), (5.9, 2, 127), (0.3, 2, 123), (3.0e38, 2, 252),
])
def test_mx_shared_scale_rule(orc, amax, fmt, code):
    """E8M0 scale = floor(log2(amax)) - emax + 127, emax 8 (E4M3) or 2 (E2M1):
    one block whose SwiGLU output has exactly that amax."""
    # silu(g) * u with g large: silu(g) == g, so y = g * u exactly
    I = 32
    g = np.full(I, 64.0, np.float32)
    u = np.zeros(I, np.float32)
    u[0] = amax / 64.0
    row = bf16_bits(np.concatenate([g, u]))[None, :]
    amax_bf = float(f32(row[0, I]) * 64.0)
    codes, scales = orc.swiglu_quant(row, np.array([0], np.int32), fmt)
    want = orc.lib().orc_e8m0_from_exponent(math.floor(math.log2(amax_bf)) - (8 if fmt == 1 else 2))
    assert scales[0, 0] == want == code


def test_mx_element_codes_brute_force(orc):
    rng = np.random.default_rng(3)
    rows, I = 40, 128
    gu = bf16_bits(rng.standard_normal((rows, 2 * I)) * 3)
    gu[9, I + 32:I + 64] = 0                  # all-zero blocks: scale 0, codes 0
    gu[11, I + 64:I + 96] = 0
    gu[rows - 1, 2 * I - 32:] = 0             # ... the buffer's last block
    gu[12, I:I + 32] = bf16_bits(np.full(32, 1e-39))   # tiny block: the scale clamps
    src = np.arange(rows, dtype=np.int32)
    src[5] = -1
    gf, uf = f32(gu[:, :I]), f32(gu[:, I:])
    y = np.array([[orc.lib().orc_silu(float(a)) for a in r] for r in gf], np.float32) * uf
    codes4, vals4 = e4m3_table()
    c2 = np.array([c for c, _ in E2M1])
    v2 = np.array([v for _, v in E2M1])
    for fmt in (1, 2):
        codes, scales = orc.swiglu_quant(gu, src, fmt)
        emax = 8 if fmt == 1 else 2
        for r in range(rows):
            if src[r] < 0:
                assert not codes[r].any() and not scales[r].any()
                continue
            for b in range(I // 32):
                blk = y[r, 32 * b:32 * b + 32]
                amax = np.abs(blk).max()
                if amax == 0:
                    w = 32 if fmt == 1 else 16
                    assert scales[r, b] == 0 and not codes[r, w * b:w * b + w].any()
                    continue
                # E8M0 holds 2^-127 .. 2^127: a smaller X takes the smallest scale
                X = max(math.floor(math.log2(amax)) - emax, -127)
                assert scales[r, b] == X + 127
                v = (blk.astype(np.float64) * 2.0 ** -X).astype(np.float32)
                if fmt == 1:
                    mag = brute_nearest_even(v, codes4, vals4, 0x7E)
                    want = mag | np.where(np.signbit(v), 0x80, 0)
                    assert np.array_equal(codes[r, 32 * b:32 * b + 32], want)
                else:
                    mag = brute_nearest_even(v, c2, v2, 7)
                    c = mag | np.where(np.signbit(v), 8, 0)
                    assert np.array_equal(codes[r, 16 * b:16 * b + 16], c[0::2] | (c[1::2] << 4))
        assert scales[12, 0] == 0 and 0 < np.abs(y[12, :32]).max() < 2.0 ** (-127 + emax)


def test_nvfp4_matches_dispatch_rule_on_swiglu_output(orc):
    """With g large (silu(g) == g) and u = y / g (exact: g is a power of two),
    the SwiGLU NVFP4 path must quantise y exactly as the dispatch quantises
    a row equal to y."""
    rng = np.random.default_rng(4)
    I, rows = 64, 6
    y_bf = bf16_bits(rng.standard_normal((rows, I)))
    y_bf[2, 16:32] = 0                        # an all-zero 16-element block
    g = np.full((rows, I), 64.0, np.float32)
    u = f32(y_bf) / np.float32(64.0)          # exact: power-of-two scaling
    gu = bf16_bits(np.concatenate([g, u], axis=1))
    codes, scales = orc.swiglu_quant(gu, np.arange(rows, dtype=np.int32), 0, global_scale=0.01)
    q, s = orc.permute_nvfp4(y_bf, np.arange(rows, dtype=np.int32), 0.01)
    assert np.array_equal(codes, q) and np.array_equal(scales, s)
    assert scales[2, 1] == 0 and not codes[2, 8:16].any()


def test_interleaved_equals_split(orc):
    rng = np.random.default_rng(5)
    rows, I = 10, 96
    gu = bf16_bits(rng.standard_normal((rows, 2 * I)))
    inter = np.empty_like(gu)
    inter[:, 0::2], inter[:, 1::2] = gu[:, :I], gu[:, I:]
    src = np.arange(rows, dtype=np.int32)
    for fmt in (0, 1, 2):
        a = orc.swiglu_quant(gu, src, fmt, global_scale=0.05)
        b = orc.swiglu_quant(inter, src, fmt, interleaved=True, global_scale=0.05)
        assert np.array_equal(a[0], b[0]) and np.array_equal(a[1], b[1])
