"""Pins of the oracle's GEMM scale-factor layout (no GPU): block scales of a [rows, nb]
matrix in 128 x 4 tiles of 512 bytes, entry (r, c) of a tile at (r % 32) * 16 +
(r / 32) * 4 + c. The layout is checked against a second formulation (a reshape /
transpose of the padded matrix: rows split as (tile, 4, 32), columns as (tile, 4), the
32-row and 4-row axes swapped), as a bijection, and at hand-computed positions. The
GPU test that a block-scaled GEMM reads these bytes correctly is in
tests/test_gpu_gemm_operands.py."""

import numpy as np
import pytest

import oracle


def _by_reshape(s):
    rows, nb = s.shape
    R, C = -(-rows // 128) * 128, -(-nb // 4) * 4
    p = np.zeros((R, C), np.uint8)
    p[:rows, :nb] = s
    # [tile_r, r/32, r%32, tile_c, c] -> [tile_r, tile_c, r%32, r/32, c]
    t = p.reshape(R // 128, 4, 32, C // 4, 4).transpose(0, 3, 2, 1, 4)
    return t.reshape(-1)


@pytest.mark.parametrize("rows,nb", [(1, 1), (128, 4), (130, 7), (300, 128), (4096, 344)])
def test_layout_matches_reshape_form_and_round_trips(rows, nb):
    g = np.random.default_rng(rows * 1000 + nb)
    s = g.integers(0, 255, size=(rows, nb), dtype=np.uint8)
    out = oracle.scales_to_gemm(s, rows, nb)
    assert out.size == -(-rows // 128) * 128 * (-(-nb // 4) * 4)
    assert np.array_equal(out, _by_reshape(s))
    assert np.array_equal(oracle.scales_from_gemm(out, rows, nb), s)


def test_layout_hand_positions():
    nb = 8                                   # two tiles per tile row
    assert oracle.gemm_scale_offset(0, 0, nb) == 0
    assert oracle.gemm_scale_offset(0, 3, nb) == 3
    assert oracle.gemm_scale_offset(1, 0, nb) == 16
    assert oracle.gemm_scale_offset(31, 0, nb) == 31 * 16
    assert oracle.gemm_scale_offset(32, 0, nb) == 4
    assert oracle.gemm_scale_offset(127, 3, nb) == 31 * 16 + 3 * 4 + 3
    assert oracle.gemm_scale_offset(0, 4, nb) == 512
    assert oracle.gemm_scale_offset(128, 0, nb) == 1024
    assert oracle.gemm_scale_offset(129, 5, nb) == 1024 + 512 + 16 + 1


def test_layout_is_a_bijection_on_the_padded_matrix():
    rows, nb = 256, 12
    offs = {oracle.gemm_scale_offset(r, c, nb) for r in range(rows) for c in range(nb)}
    assert len(offs) == rows * nb and max(offs) < oracle.gemm_scale_bytes(rows, nb)
