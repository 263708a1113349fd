"""Pins for the oracle's backward pass (CPU only): adjoint identities in
float64 (the dispatch and combine are linear in their data, so
<forward(x), g> == <x, backward(g)>), the k = 1 special case, and a closed
form for the gate gradient."""
import numpy as np
import torch

from combine_topk_ids_scan_b200.inputs import make_workload


def f32(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


def bf16_bits(x):
    return torch.from_numpy(np.asarray(x, np.float32)).to(torch.bfloat16).view(
        torch.int16).numpy().view(np.uint16)


def _setup(orc, n_tokens=256, cfg="mid_zipf", C_extra=37):
    w = make_workload(cfg, n_tokens=n_tokens)
    C = w.N * w.k + C_extra                          # some padding rows
    lay = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C)
    rng = np.random.default_rng(17)
    g_rows = bf16_bits(rng.standard_normal((C, w.H)))
    g_tok = bf16_bits(rng.standard_normal((w.N, w.H)))
    X = bf16_bits(rng.standard_normal((C, w.H)))
    return w, lay, g_rows, g_tok, X


def test_permute_backward_is_the_adjoint(orc):
    w, lay, g_rows, _, _ = _setup(orc)
    gh = orc.permute_backward(g_rows, lay.pair_slot)
    x = f32(w.hidden).astype(np.float64)
    fwd = f32(orc.permute_bf16(w.hidden, lay.row_src)).astype(np.float64)
    lhs = np.sum(fwd * f32(g_rows).astype(np.float64))
    rhs = np.sum(x * f32(gh).astype(np.float64))
    # gh is rounded once to bf16: relative error <= 2^-8 per element
    bound = 2.0 ** -8 * np.sum(np.abs(x) * np.abs(f32(gh))) + 1e-9
    assert abs(lhs - rhs) <= bound


def test_permute_backward_k1_is_a_gather(orc):
    rng = np.random.default_rng(2)
    g = bf16_bits(rng.standard_normal((50, 32)))
    slots = rng.permutation(50)[:40].astype(np.int32).reshape(40, 1)
    slots[3, 0] = -1
    gh = orc.permute_backward(g, slots)
    want = np.where(slots >= 0, g[np.maximum(slots[:, 0], 0)], 0)
    assert np.array_equal(gh, want)


def test_combine_backward_adjoint_in_expert_outputs(orc):
    w, lay, _, g_tok, X = _setup(orc)
    gx, _ = orc.combine_backward(g_tok, X, w.gates, lay.pair_slot)
    # y = combine(X) in float64 (a second formulation of the forward)
    xf = f32(X).astype(np.float64)
    y = np.zeros((w.N, w.H))
    for j in range(w.k):
        s = lay.pair_slot[:, j]
        y += np.where(s[:, None] >= 0, w.gates[:, j:j + 1].astype(np.float64) * xf[s], 0)
    lhs = np.sum(y * f32(g_tok).astype(np.float64))
    rhs = np.sum(xf * f32(gx).astype(np.float64))
    bound = 2.0 ** -8 * np.sum(np.abs(xf) * np.abs(f32(gx))) + 1e-9
    assert abs(lhs - rhs) <= bound
    # rows no pair owns carry no gradient
    assert np.all(gx[lay.row_src < 0] == 0)


def test_permute_backward_exact_on_integer_rows(orc):
    """Integer gradients with |g| <= 16: every partial sum of k = 6 terms is
    exact in fp32 and the total (|sum| <= 96) exact in bf16, so the dispatch
    backward must equal numpy's gather-sum bit for bit; masked slots and a
    slot equal to rows contribute nothing."""
    w = make_workload("mid_zipf", n_tokens=256)
    C = w.N * w.k + 37
    lay = orc.layout(w.ids, w.E, w.S, w.H, recv_capacity=C)
    H = 256                                   # any row width; keeps the test small
    rng = np.random.default_rng(21)
    g = rng.integers(-16, 17, size=(C, H)).astype(np.float32)
    slots = lay.pair_slot.copy()
    slots[0, 1] = C                           # == rows: outside the buffer
    slots[1, 2] = -1
    gh = orc.permute_backward(bf16_bits(g), slots)
    valid = (slots >= 0) & (slots < C)
    want = np.where(valid[:, :, None], g[np.clip(slots, 0, C - 1)], 0).sum(axis=1)
    assert np.array_equal(f32(gh), want.astype(np.float32))


def test_combine_backward_exact_on_integer_rows(orc):
    """Power-of-two gates and small integer rows make every product and dot
    exact: grad_expert_out[slot(t,j)] = w[t,j] * grad_y[t] and
    grad_gates[t,j] = <grad_y[t], X[slot(t,j)]> (numpy einsum), zeros in the
    rows no pair owns, gate gradient 0 for a masked slot or a slot equal to
    rows."""
    N, k, H, rows = 40, 4, 96, 200
    rng = np.random.default_rng(22)
    slots = (1 + rng.permutation(rows - 1)[:N * k]).astype(np.int32).reshape(N, k)
    slots[3, 0] = -1
    slots[7, 2] = rows
    gates = (2.0 ** rng.integers(-3, 3, size=(N, k))).astype(np.float32)
    gy = rng.integers(-8, 9, size=(N, H)).astype(np.float32)
    X = rng.integers(-8, 9, size=(rows, H)).astype(np.float32)
    gx, gw = orc.combine_backward(bf16_bits(gy), bf16_bits(X), gates, slots)
    valid = (slots >= 0) & (slots < rows)
    want_gx = np.zeros((rows, H), np.float32)
    t_idx, j_idx = np.nonzero(valid)
    want_gx[slots[t_idx, j_idx]] = gates[t_idx, j_idx, None] * gy[t_idx]
    assert np.array_equal(f32(gx), want_gx)
    want_gw = np.einsum("th,tjh->tj", gy.astype(np.float64),
                        X[np.clip(slots, 0, rows - 1)].astype(np.float64))
    want_gw = np.where(valid, want_gw, 0.0).astype(np.float32)
    assert np.array_equal(gw, want_gw)


def test_gate_gradient_closed_form(orc):
    """With constant expert rows X[s] = c_s and grad_y[t] = 1, the gate
    gradient is H * c_s exactly."""
    N, k, H = 20, 3, 64
    rng = np.random.default_rng(4)
    c = np.array([0.5, -1.25, 2.0, 3.0, -0.75, 1.5], np.float32)
    X = bf16_bits(np.repeat(c[:, None], H, axis=1))
    slots = rng.integers(-1, 6, size=(N, k)).astype(np.int32)
    gates = rng.random((N, k)).astype(np.float32)
    gy = bf16_bits(np.ones((N, H)))
    _, gw = orc.combine_backward(gy, X, gates, slots)
    want = np.where(slots >= 0, H * c[np.maximum(slots, 0)], 0).astype(np.float32)
    assert np.array_equal(gw, want)
