"""Pins for the oracle's permute (bf16 / block FP8 / NVFP4) and combine.

Checked against: numpy fancy indexing (the bf16 gather), brute-force
nearest-even searches over the format tables (independent of the oracle's
converters), hand-worked blocks, dequantisation error bounds, a float64
weighted sum, closed forms (k=1 gather, identity-expert round trip).
"""
import numpy as np
import pytest
import torch

from combine_topk_ids_scan_b200.inputs import make_workload
from test_oracle_formats import E2M1, brute_nearest_even, e4m3_table


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


@pytest.fixture(scope="module")
def tiny(orc):
    w = make_workload("tiny")
    lay = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=w.recv_capacity)
    return w, lay


def test_permute_bf16_is_a_gather_with_zero_padding(orc):
    rng = np.random.default_rng(5)
    hidden = rng.integers(0, 2**16, size=(37, 64)).astype(np.uint16)
    row_src = rng.integers(-1, 37, size=91).astype(np.int32)
    out = orc.permute_bf16(hidden, row_src)
    want = np.where(row_src[:, None] >= 0, hidden[np.maximum(row_src, 0)], 0)
    assert np.array_equal(out, want)


def _dec_e4m3(codes):
    return torch.from_numpy(np.asarray(codes, np.uint8)).view(torch.float8_e4m3fn).float().numpy()


def test_permute_fp8_against_brute_force(orc, tiny):
    w, lay = tiny
    hidden = w.hidden.copy()
    hidden[3, 128:256] = 0                    # an all-zero block
    hidden[5, :] = bf16_bits(f32(hidden[5]) * 100)  # an outlier row
    row_src = lay.row_src.copy()
    row_src[7] = -1                            # a padding row
    q, sc = orc.permute_fp8(hidden, row_src)
    codes, vals = e4m3_table()
    x = f32(hidden[np.maximum(row_src, 0)]).reshape(len(row_src), -1, 128)
    amax = np.abs(x).max(axis=2)
    # scale: the decode multiplier amax / 448, one fp32 rounding
    want_sc = np.where(amax > 0, amax / np.float32(448.0), 0).astype(np.float32)
    want_sc[row_src < 0] = 0
    assert np.array_equal(sc, want_sc)
    # codes: brute-force nearest-even of x / scale (fp32 division)
    v = (x / np.where(want_sc > 0, want_sc, 1)[:, :, None]).astype(np.float32)
    mag = brute_nearest_even(v.reshape(-1), codes, vals, 0x7E)
    want_q = (mag | np.where(np.signbit(v.reshape(-1)), 0x80, 0)).reshape(q.shape)
    want_q[np.repeat(want_sc == 0, 128, axis=1)] = 0
    assert np.array_equal(q.astype(np.int64), want_q)
    # the block maximum lands on +-448 and dequantisation error is <= half an ulp
    live = want_sc > 0
    qb = q.reshape(len(row_src), -1, 128)
    assert np.all((np.abs(_dec_e4m3(qb)).max(axis=2) == 448)[live])
    sc64 = want_sc.astype(np.float64)[:, :, None]
    deq = _dec_e4m3(qb).astype(np.float64) * sc64
    e = np.floor(np.log2(np.maximum(np.abs(v), 2.0**-6)))
    half_ulp = 2.0 ** (e - 4) * sc64
    # half an E4M3 ulp of x/scale, plus the fp32 rounding of the quotient
    bound = half_ulp + 2.0**-23 * np.abs(x.astype(np.float64))
    assert np.all((np.abs(deq - x) <= bound)[live])
    assert np.all(q[7] == 0) and np.all(sc[7] == 0)


@pytest.mark.parametrize("last", ["padding", "zero_block"])
def test_permute_quantisers_fill_to_the_end_of_the_buffer(orc, last):
    """The buffer's last row as a padding row, or as a row ending in an
    all-zero block: its codes and scales are all zero up to the end of the
    buffer and not a byte further (every oracle output is followed by a
    guard that the call checks)."""
    rng = np.random.default_rng(8)
    H = 256
    hidden = bf16_bits(rng.standard_normal((4, H)))
    hidden[1, H - 128:] = 0                   # the last 128 elements are zero
    row_src = np.array([0, 2, -1 if last == "padding" else 1], np.int32)
    for name, (q, sc), block in (("fp8", orc.permute_fp8(hidden, row_src), 128),
                                 ("nvfp4", orc.permute_nvfp4(hidden, row_src, 0.01), 16),
                                 ("mxfp4", orc.permute_mxfp4(hidden, row_src), 32)):
        code_bytes = q.shape[1] // (H // 128)        # code bytes of the last 128 elements
        assert not q[2, -code_bytes:].any(), name
        assert not sc[2, -(128 // block):].any(), name
        if last == "padding":
            assert not q[2].any() and not sc[2].any(), name
        else:
            assert q[2, :-code_bytes].any(), name


def test_permute_nvfp4_hand_block(orc):
    # one row, H=32: block 0 = [6, 0.5, 0, ...], block 1 = [-3, 1.5, 0, ...]
    x = np.zeros((1, 32), np.float32)
    x[0, 0], x[0, 1] = 6.0, 0.5
    x[0, 16], x[0, 17] = -3.0, 1.5
    q, sc = orc.permute_nvfp4(bf16_bits(x), np.array([0], np.int32), 1.0)
    # block 0: amax 6 -> (6/6)/1 = 1.0 -> scale code 0x38, d = 1: codes 7 | 1<<4
    assert sc[0, 0] == 0x38 and q[0, 0] == 0x17 and np.all(q[0, 1:8] == 0)
    # block 1: amax 3 -> 0.5 -> scale code 0x30, d = 0.5: -3/.5=-6 -> 0xF, 1.5/.5=3 -> 5
    assert sc[0, 1] == 0x30 and q[0, 8] == 0x5F
    # an all-zero block: the scale code and the payload are 0
    q, sc = orc.permute_nvfp4(bf16_bits(np.zeros((1, 16))), np.array([0], np.int32), 0.37)
    assert sc[0, 0] == 0 and np.all(q == 0)


def test_permute_nvfp4_against_brute_force(orc, tiny):
    w, lay = tiny
    row_src = lay.row_src.copy()
    row_src[2] = -1
    q, sc = orc.permute_nvfp4(w.hidden, row_src, w.global_scale)
    gs = np.float32(w.global_scale)
    codes4, vals4 = e4m3_table()
    c2 = np.array([c for c, _ in E2M1])
    v2 = np.array([v for _, v in E2M1])
    x = f32(w.hidden[np.maximum(row_src, 0)]).reshape(len(row_src), -1, 16)
    amax = np.abs(x).max(axis=2)
    s_f = ((amax / np.float32(6.0)).astype(np.float32) / gs).astype(np.float32)
    want_sc = brute_nearest_even(s_f.reshape(-1), codes4, vals4, 0x7E).reshape(s_f.shape)
    want_sc[row_src < 0] = 0
    assert np.array_equal(sc.astype(np.int64), want_sc)
    d = (_dec_e4m3(want_sc.astype(np.uint8)) * gs).astype(np.float32)
    v = (x / np.where(d > 0, d, 1)[:, :, None]).astype(np.float32)
    mag = brute_nearest_even(v.reshape(-1), c2, v2, 7)
    code = (mag | np.where(np.signbit(v.reshape(-1)), 8, 0)).reshape(x.shape)
    code[np.broadcast_to((d == 0)[:, :, None], code.shape)] = 0
    code[row_src < 0] = 0
    code = code.reshape(len(row_src), -1)
    want_q = (code[:, 0::2] | (code[:, 1::2] << 4))
    assert np.array_equal(q.astype(np.int64), want_q)
    assert np.all(q[2] == 0)


def _combine_f64(X, gates, slots):
    xf = f32(X).astype(np.float64)
    N, k = slots.shape
    acc = np.zeros((N, X.shape[1]))
    mag = np.zeros_like(acc)
    for j in range(k):
        s = slots[:, j]
        ok = s >= 0
        term = gates[:, j:j + 1].astype(np.float64) * xf[np.maximum(s, 0)]
        acc += np.where(ok[:, None], term, 0)
        mag += np.where(ok[:, None], np.abs(term), 0)
    return acc, mag


def test_combine_within_one_bf16_ulp_of_exact(orc, tiny):
    w, lay = tiny
    y = orc.combine(w.expert_out, w.gates, lay.pair_slot)
    exact, mag = _combine_f64(w.expert_out, w.gates, lay.pair_slot)
    got = f32(y).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0**-126))) - 7)
    assert np.all(np.abs(got - exact) <= ulp + w.k * 2.0**-23 * mag)


def test_combine_k1_unit_gate_is_gather(orc):
    rng = np.random.default_rng(9)
    X = bf16_bits(rng.standard_normal((20, 48)))
    slots = rng.integers(-1, 20, size=(30, 1)).astype(np.int32)
    y = orc.combine(X, np.ones((30, 1), np.float32), slots)
    want = np.where(slots >= 0, X[np.maximum(slots[:, 0], 0)], 0)
    # a masked pair leaves the +0 accumulator
    assert np.array_equal(y, want)


def test_combine_skips_masked_and_out_of_range(orc):
    # X is the first 3 rows of a 4-row array: a read of row 3 would see
    # non-zero values
    X4 = bf16_bits(np.arange(1, 17, dtype=np.float32).reshape(4, 4))
    X = X4[:3]
    gates = np.array([[0.5, 0.25, 2.0, 4.0]], np.float32)
    slots = np.array([[1, -1, 7, 3]], np.int32)   # rows 7 and 3 (= rows) do not exist
    y = orc.combine(X, gates, slots)
    assert np.array_equal(f32(y[0]), np.float32(0.5) * f32(X[1]))


def test_identity_expert_round_trip(orc, tiny):
    """combine(dispatch(x)) == x bit-exactly when every expert is the
    identity and each token's gates sum to 1 (softmax)."""
    w, lay = tiny
    disp = orc.permute_bf16(w.hidden, lay.row_src)
    y = orc.combine(disp, w.gates, lay.pair_slot)
    assert np.array_equal(y, w.hidden)


def test_capacity_mode_round_trip_drops(orc):
    w = make_workload("decode_capacity", n_tokens=64, with_expert_out=False)
    lay = orc.layout(w.ids, w.E, w.S, w.H, expert_capacity=2)
    assert lay.drop_mask.sum() > 0
    disp = orc.permute_bf16(w.hidden, lay.row_src)
    y = orc.combine(disp, w.gates, lay.pair_slot)
    # kept-gate sum scales the token; no renormalisation after drops
    keep = (lay.pair_slot >= 0)
    gsum = np.where(keep, w.gates, 0).astype(np.float64).sum(axis=1)
    exact = f32(w.hidden).astype(np.float64) * gsum[:, None]
    got = f32(y).astype(np.float64)
    ulp = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0**-126))) - 7)
    assert np.all(np.abs(got - exact) <= ulp + 8 * 2.0**-23 * np.abs(exact))
