"""Pins for the oracle's pre-multiplied-gates dispatch (CPU only).

DeepSpeed v0.19.4 function list: token representations pre-multiplied by
their router scores before expert compute.  The dispatch writes
bf16(w[t,j] * x[t]) to pair (t, j)'s row; the combine of that variant is the
unweighted sum, and its backward is the weighted combine (gradient of x) plus
a dot product (gradient of the gates).  Checked against torch's fp32 product
and bf16 cast, the plain dispatch (unit gates), and exact integer-valued
cases of the variant's forward and backward identities.
"""
import numpy as np
import torch

from combine_topk_ids_scan_b200.inputs import make_workload


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _layout(orc, cfg="mid_zipf", n_tokens=256, extra=37):
    w = make_workload(cfg, n_tokens=n_tokens)
    C = w.N * w.k + extra
    return w, orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C), C


def test_matches_torch_product_and_cast(orc):
    w, lay, C = _layout(orc)
    out = orc.permute_premultiplied(w.hidden, w.gates, lay.pair_slot, C)
    x = torch.from_numpy(w.hidden.view(np.int16)).view(torch.bfloat16).float()
    g = torch.from_numpy(w.gates)
    prod = (g[:, :, None] * x[:, None, :]).to(torch.bfloat16).view(torch.int16).numpy()
    want = np.zeros((C, w.H), np.uint16)
    t_idx, j_idx = np.nonzero(lay.pair_slot >= 0)
    want[lay.pair_slot[t_idx, j_idx]] = prod.view(np.uint16)[t_idx, j_idx]
    assert np.array_equal(out, want)
    assert not out[lay.row_src < 0].any()


def test_hand_slots_unowned_rows_and_bounds(orc):
    """Hand-made slots: rows 0, 4, 5 and 6 owned by no pair (zeros), a masked
    pair, a slot equal to rows (skipped), and a valid-looking row of slots,
    gates and tokens just past the end of each input, so that a read past
    pair_slot, gates or hidden would change the output."""
    H, rows = 16, 8
    x_full = bf16_bits(np.arange(1, 4 * H + 1, dtype=np.float32).reshape(4, H))
    g_full = np.array([[0.5, 2.0], [4.0, 0.25], [1.5, 3.0], [8.0, 8.0]], np.float32)
    s_full = np.array([[1, 2], [-1, 7], [3, rows], [0, 0]], np.int32)
    out = orc.permute_premultiplied(x_full[:3], g_full[:3], s_full[:3], rows)
    want = np.zeros((rows, H), np.uint16)
    for t, j in ((0, 0), (0, 1), (1, 1), (2, 0)):
        want[s_full[t, j]] = bf16_bits(g_full[t, j] * f32(x_full[t]))
    assert np.array_equal(out, want)


def test_unit_gates_is_the_plain_dispatch(orc):
    w, lay, C = _layout(orc, "tiny", n_tokens=None, extra=5)
    out = orc.permute_premultiplied(w.hidden, np.ones_like(w.gates), lay.pair_slot, C)
    assert np.array_equal(out, orc.permute_bf16(w.hidden, lay.row_src))


def test_capacity_drops_and_masked_pairs(orc):
    w = make_workload("decode_capacity", n_tokens=64, with_expert_out=False)
    lay = orc.layout(w.ids, w.E, w.S, w.H, expert_capacity=2)
    rows = w.E * 2
    out = orc.permute_premultiplied(w.hidden, w.gates, lay.pair_slot, rows)
    assert lay.drop_mask.sum() > 0
    assert not out[lay.row_src < 0].any()
    kept = np.nonzero(lay.pair_slot >= 0)
    g = lay.pair_slot[kept]
    x = f32(w.hidden)[kept[0]]
    want = bf16_bits(w.gates[kept][:, None] * x)
    assert np.array_equal(out[g], want)


def test_variant_identities_exact_on_integer_rows(orc):
    """Small integers and power-of-two gates make every product and sum
    exact, so the variant's identities hold bit for bit:
      forward:  unweighted sum of D_w x  ==  weighted combine of D x;
      backward: <D_w x, g> == <x, combine_w(g)> (the gradient of x is the
                weighted combine) and d/dw[t,j] <D_w x, g> = <x[t], g[slot]>
                (the combine backward's gate gradient with the roles of its
                inputs swapped) == numpy einsum."""
    w, lay, C = _layout(orc, "mid_zipf", 256, 37)
    H = 128
    rng = np.random.default_rng(31)
    x = rng.integers(-8, 9, size=(w.N, H)).astype(np.float32)
    g = rng.integers(-8, 9, size=(C, H)).astype(np.float32)
    gates = (2.0 ** rng.integers(-2, 2, size=(w.N, w.k))).astype(np.float32)
    xb, gb = bf16_bits(x), bf16_bits(g)
    dwx = orc.permute_premultiplied(xb, gates, lay.pair_slot, C)
    # forward: the variant's combine (unweighted) == the plain weighted combine
    y_variant = orc.permute_backward(dwx, lay.pair_slot)
    y_plain = orc.combine(orc.permute_bf16(xb, lay.row_src), gates, lay.pair_slot)
    assert np.array_equal(y_variant, y_plain)
    # backward in x: the adjoint of D_w is the weighted combine
    lhs = np.sum(f32(dwx).astype(np.float64) * g)
    rhs = np.sum(x.astype(np.float64) * f32(orc.combine(gb, gates, lay.pair_slot)))
    assert lhs == rhs
    # backward in the gates: <x[t], g[slot(t,j)]>
    _, gw = orc.combine_backward(xb, gb, gates, lay.pair_slot)
    valid = lay.pair_slot >= 0
    want = np.einsum("th,tjh->tj", x.astype(np.float64),
                     g[np.maximum(lay.pair_slot, 0)].astype(np.float64))
    assert np.array_equal(gw, np.where(valid, want, 0).astype(np.float32))
