"""Pins of the raster <-> Z-order permutation (Step 5: Index Reordering for
Images): a hand-written grid, a hand-decoded token, the tile structure the
pooling relies on, and round trips."""

import numpy as np
import pytest

import oracle


def test_zorder_of_a_4x4_grid_written_out():
    # x bit 0 -> token bit 0, y bit 0 -> bit 1, x bit 1 -> bit 2, y bit 1 -> bit 3
    want = np.array([[0, 1, 4, 5],
                     [2, 3, 6, 7],
                     [8, 9, 12, 13],
                     [10, 11, 14, 15]])
    assert np.array_equal(oracle.zorder_index(4, 4).reshape(4, 4), want)


def test_a_token_decoded_by_hand():
    # token 54 = 0b110110: even bits (0,1,1) -> x = 6, odd bits (1,0,1) -> y = 5
    z = oracle.zorder_index(8, 8)
    assert z[5 * 8 + 6] == 54


@pytest.mark.parametrize("side", [8, 16, 32])
def test_runs_of_16_tokens_are_4x4_tiles(side):
    z = oracle.zorder_index(side, side)
    inv = np.argsort(z)  # raster position of each Z token
    ys, xs = inv // side, inv % side
    for t0 in range(0, side * side, 16):
        x, y = xs[t0:t0 + 16], ys[t0:t0 + 16]
        assert x.max() - x.min() == 3 and y.max() - y.min() == 3
        assert x.min() % 4 == 0 and y.min() % 4 == 0
    # and runs of 256 tokens are 16x16 tiles (the level-2 tokens)
    if side >= 16:
        for t0 in range(0, side * side, 256):
            x, y = xs[t0:t0 + 256], ys[t0:t0 + 256]
            assert x.max() - x.min() == 15 and y.max() - y.min() == 15


def test_is_a_permutation_and_round_trips():
    z = oracle.zorder_index(16, 16)
    assert np.array_equal(np.sort(z), np.arange(256))
    rng = np.random.default_rng(5)
    X = rng.standard_normal((2, 3, 256, 8))
    Zx = oracle.reorder(X, 16, 16, to_zorder=True)
    assert np.array_equal(oracle.reorder(Zx, 16, 16, to_zorder=False), X)
    # the raster pixel (x, y) lands at its Z token
    assert np.array_equal(Zx[:, :, z[3 * 16 + 7]], X[:, :, 3 * 16 + 7])


def test_non_square_images_are_rejected():
    with pytest.raises(ValueError):
        oracle.zorder_index(8, 16)
    with pytest.raises(ValueError):
        oracle.zorder_index(12, 12)
