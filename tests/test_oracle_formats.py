"""Pins for the oracle's number formats (CPU only).

The oracle's converters are checked against things that are not the oracle:
torch's own bfloat16 / float8_e4m3fn casts, the OCP format tables in
tests/golden, and a brute-force nearest-value search (ties to the even code)
over those tables.
"""
import os

import numpy as np
import pytest
import torch

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_table(name):
    rows = []
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if not line or line.startswith("#"):
            continue
        c, v = line.split()
        rows.append((int(c, 16), float(v)))
    return rows


def brute_nearest_even(v, codes, values, max_code):
    """Nearest table value to |v| (ties to the even code), saturating at the
    table maximum; codes/values are the non-negative finite codes."""
    v = np.asarray(v, np.float64)
    a = np.abs(v)
    d = np.abs(a[:, None] - values[None, :])
    best = d.min(axis=1, keepdims=True)
    cand = d == best
    # among tied candidates prefer an even code
    even = (codes[None, :] % 2) == 0
    pick_even = cand & even
    has_even = pick_even.any(axis=1)
    idx = np.where(has_even, pick_even.argmax(axis=1), cand.argmax(axis=1))
    out = codes[idx].astype(np.int64)
    out[a > values.max()] = max_code
    return out


def e4m3_table():
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    codes = np.arange(0, 0x7F)          # non-negative finite codes 0x00..0x7E
    return codes, dec[codes].astype(np.float64)


E2M1 = _read_table("e2m1_values.txt")


# ------------------------------------------------------------------ bf16
def test_bf16_matches_torch_cast(orc):
    rng = np.random.default_rng(1)
    x = np.concatenate([
        rng.standard_normal(200000).astype(np.float32),
        (rng.standard_normal(20000) * 1e30).astype(np.float32),
        (rng.standard_normal(20000) * 1e-38).astype(np.float32),   # subnormals
        np.array([0.0, -0.0, 3.3895314e38, -3.3895314e38, 1.0 + 2**-8, 1.0 + 3 * 2**-8,
                  1.0 + 2**-8 + 2**-20], np.float32),
    ])
    # exact ties on the dropped half, both parities
    bits = rng.integers(0, 2**31, 20000, dtype=np.uint64).astype(np.uint32)
    bits = (bits & np.uint32(0xFFFF0000)) | np.uint32(0x8000)
    bits = bits[((bits >> 23) & 0xFF) != 0xFF]
    x = np.concatenate([x, bits.view(np.float32)])
    want = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    got = orc.bf16_from_f32(x)
    assert np.array_equal(got, want)


def test_bf16_infinities_and_nans(orc):
    """IEEE 754: an infinity converts to the infinity of the same sign; a NaN
    stays a NaN (all-ones exponent, non-zero fraction) with its sign, whatever
    its payload (the payload itself is not pinned)."""
    got = orc.bf16_from_f32(np.array([np.inf, -np.inf], np.float32))
    assert got.tolist() == [0x7F80, 0xFF80]
    nan_bits = np.array([0x7FC00000, 0x7F800001, 0xFF800001, 0x7FFFFFFF, 0x7F80FFFF,
                         0xFFC12345, 0x7F810000], np.uint32)
    got = orc.bf16_from_f32(nan_bits.view(np.float32)).astype(np.uint32)
    assert np.all((got & 0x7F80) == 0x7F80) and np.all((got & 0x7F) != 0)
    assert np.array_equal(got >> 15, nan_bits >> 31)
    back = torch.from_numpy(got.astype(np.uint16).view(np.int16)).view(torch.bfloat16).float()
    assert torch.isnan(back).all()


# ------------------------------------------------------------------ e4m3
def test_e4m3_decode_matches_torch_and_spec(orc):
    dec = torch.arange(256, dtype=torch.uint8).view(torch.float8_e4m3fn).float().numpy()
    for c in range(256):
        v = orc.e4m3_to_f32(c)
        if np.isnan(dec[c]):
            assert np.isnan(v)
        else:
            assert v == dec[c] and np.signbit(v) == np.signbit(dec[c]), c
    for c, v in _read_table("e4m3_points.txt"):
        got = orc.e4m3_to_f32(c)
        assert got == v and np.signbit(got) == np.signbit(v), (hex(c), got, v)


def test_e4m3_encode_matches_torch_in_range(orc):
    codes, vals = e4m3_table()
    rng = np.random.default_rng(2)
    mids = (vals[1:] + vals[:-1]) / 2          # every midpoint between codes
    x = np.concatenate([
        vals, mids, np.nextafter(mids.astype(np.float32), np.float32(0)),
        np.nextafter(mids.astype(np.float32), np.float32(1000)),
        rng.uniform(-463, 463, 200000), rng.standard_normal(100000) * 1e-3,
    ]).astype(np.float32)
    x = np.concatenate([x, -x])
    x = x[np.abs(x) < 464]                     # torch turns >= 464 into NaN
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_from_f32(x)
    assert np.array_equal(got, want)


def test_e4m3_encode_nan(orc):
    """E4M3 ("fn") keeps one NaN encoding, S.1111.111: a NaN of either sign
    and any payload maps to it with its sign, as torch's cast does."""
    nan_bits = np.array([0x7FC00000, 0xFFC00000, 0x7F800001, 0xFF812345, 0x7FFFFFFF], np.uint32)
    x = nan_bits.view(np.float32)
    want = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = orc.e4m3_from_f32(x)
    assert np.array_equal(got, want) and np.array_equal(got, [0x7F, 0xFF, 0x7F, 0xFF, 0x7F])


def test_e4m3_encode_brute_force_and_saturation(orc):
    codes, vals = e4m3_table()
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.uniform(0, 600, 20000), rng.uniform(0, 0.02, 20000),
                        (vals[1:] + vals[:-1]) / 2, [448.0, 449.0, 464.0, 1e9, 3.4e38]])
    x = x.astype(np.float32)
    want = brute_nearest_even(x, codes, vals, 0x7E)
    assert np.array_equal(orc.e4m3_from_f32(x).astype(np.int64), want)
    neg = orc.e4m3_from_f32(-x)
    assert np.array_equal(neg.astype(np.int64), want | 0x80)
    assert orc.e4m3_from_f32(np.array([-0.0], np.float32))[0] == 0x80
    assert orc.e4m3_from_f32(np.array([np.inf], np.float32))[0] == 0x7E


# ------------------------------------------------------------------ e2m1
def test_e2m1_decode_table(orc):
    assert len(E2M1) == 8
    for c, v in E2M1:
        assert orc.e2m1_to_f32(c) == v
        assert orc.e2m1_to_f32(c | 8) == -v


def test_e2m1_encode_brute_force(orc):
    codes = np.array([c for c, _ in E2M1])
    vals = np.array([v for _, v in E2M1])
    rng = np.random.default_rng(4)
    mids = (vals[1:] + vals[:-1]) / 2
    x = np.concatenate([vals, mids, rng.uniform(0, 8, 50000), rng.uniform(0, 1.2, 20000)])
    x = x.astype(np.float32)
    x = np.concatenate([x, np.nextafter(x, np.float32(0)), np.nextafter(x, np.float32(9))])
    want = brute_nearest_even(x, codes, vals, 7)
    got = orc.e2m1_from_f32(x).astype(np.int64)
    assert np.array_equal(got, want)
    assert np.array_equal(orc.e2m1_from_f32(-x).astype(np.int64), want | 8)


@pytest.mark.parametrize("v,code", [
    (0.25, 0x0), (0.75, 0x2), (1.25, 0x2), (1.75, 0x4), (2.5, 0x4), (3.5, 0x6),
    (5.0, 0x6), (5.5, 0x7), (7.0, 0x7), (1e30, 0x7), (-0.0, 0x8), (-0.25, 0x8),
    (-5.0, 0xE),
])
def test_e2m1_ties_to_even_examples(orc, v, code):
    # midpoints between adjacent E2M1 values go to the even code
    assert orc.e2m1_from_f32(np.array([v], np.float32))[0] == code
