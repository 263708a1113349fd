"""Pins for the oracle's block-scale atom layout (CPU only).

The Mojo MAX ep_comm page defines SF_ROW_STRIDE_LOCAL = SF_ATOM_M[1] * 4 and
SF_ATOM_ELEMS_LOCAL = SF_ATOM_M[0] * SF_ROW_STRIDE_LOCAL; with SF_ATOM_M read
as (32, 4), an atom holds 128 rows x 4 scale columns in 512 bytes, rows m and
m + 32 are 4 bytes apart and rows m, m + 1 are 16 bytes apart.
"""
import numpy as np
import pytest

SF_ATOM_M = (32, 4)
SF_ROW_STRIDE_LOCAL = SF_ATOM_M[1] * 4
SF_ATOM_ELEMS_LOCAL = SF_ATOM_M[0] * SF_ROW_STRIDE_LOCAL


def _positions(orc, rows, nsf):
    # mark every scale with a distinct id (mod 255, +1 so no mark is 0)
    ids = (np.arange(rows * nsf) % 255 + 1).astype(np.uint8).reshape(rows, nsf)
    return ids, orc.swizzle_scales(ids)


def test_hand_positions(orc):
    rows, nsf = 300, 9
    lin = np.zeros((rows, nsf), np.uint8)
    col_tiles = 3
    cases = {(0, 0): 0, (1, 0): 16, (32, 0): 4, (33, 2): 22, (127, 3): 511,
             (0, 4): 512, (0, 8): 1024, (128, 0): 512 * col_tiles, (129, 5): 512 * 4 + 16 + 1,
             (299, 8): 512 * (2 * col_tiles + 2) + (299 % 32) * 16 + ((299 // 32) % 4) * 4}
    for (m, c), off in cases.items():
        lin[:] = 0
        lin[m, c] = 7
        out = orc.swizzle_scales(lin)
        assert out.size == 384 * 12
        assert np.nonzero(out)[0].tolist() == [off], (m, c)


@pytest.mark.parametrize("rows,nsf", [(128, 4), (1, 1), (257, 448), (65536 // 64, 448)])
def test_bijection_and_zero_fill(orc, rows, nsf):
    ids, out = _positions(orc, rows, nsf)
    assert out.size == -(-rows // 128) * 128 * (-(-nsf // 4) * 4)
    m, c = np.meshgrid(np.arange(rows), np.arange(nsf), indexing="ij")
    col_tiles = -(-nsf // 4)
    off = ((m // 128) * col_tiles + c // 4) * SF_ATOM_ELEMS_LOCAL + \
        (m % 32) * SF_ROW_STRIDE_LOCAL + ((m // 32) % 4) * 4 + c % 4
    assert np.unique(off).size == rows * nsf                      # injective
    assert np.array_equal(out[off.reshape(-1)], ids.reshape(-1))  # right place
    mask = np.ones(out.size, bool)
    mask[off.reshape(-1)] = False
    assert np.all(out[mask] == 0)                                 # the rest is zero


def test_atom_strides_follow_the_page_formulas(orc):
    def pos(m, c):
        lin = np.zeros((128, 4), np.uint8)
        lin[m, c] = 1
        return int(np.nonzero(orc.swizzle_scales(lin))[0][0])
    assert pos(1, 0) - pos(0, 0) == SF_ROW_STRIDE_LOCAL
    assert pos(32, 0) - pos(0, 0) == 4
    assert pos(0, 1) - pos(0, 0) == 1
    assert pos(127, 3) + 1 == SF_ATOM_ELEMS_LOCAL
