"""Pins for the sliding tile attention oracle: tile centres and one-axis key sets
worked by hand from the VORTA page's formula, the block-dense property, windows of
three tiles against the tile neighbourhood of oracle.tile3d, a window covering the
grid against torch SDPA, and brute-force attention of single queries."""
import math

import numpy as np
import torch

from oracle import sta, tile3d


def _qkv(seed, n, d):
    rng = np.random.default_rng(seed)
    return tuple(rng.standard_normal((n, d)) for _ in range(3))


def test_tile_centres_by_hand():
    # t = 4: positions 0..3 -> centre 2, 4..7 -> 6, 8..11 -> 10
    assert sta.tile_centre(np.arange(12), 4).tolist() == [2] * 4 + [6] * 4 + [10] * 4
    # odd t = 3: ceil(3/2) = 2 -> centres 2, 5, 8
    assert sta.tile_centre(np.arange(9), 3).tolist() == [2] * 3 + [5] * 3 + [8] * 3


def test_one_axis_key_sets_by_hand():
    # n = 20, t = 4, W = 12 (three tiles): query at 5 (tile 1, centre 6) takes centres in (0, 12]:
    # tiles 0, 1, 2 = positions 0..11; query at 0 (centre 2): centres in (-4, 8] -> tiles 0, 1
    m = sta.axis_allowed(20, 4, 12)
    assert np.nonzero(m[5])[0].tolist() == list(range(12))
    assert np.nonzero(m[0])[0].tolist() == list(range(8))
    assert np.nonzero(m[19])[0].tolist() == list(range(12, 20))
    # W = 20 (five tiles): query at 9 (centre 10) takes centres in (0, 20] -> all five tiles
    m5 = sta.axis_allowed(20, 4, 20)
    assert np.nonzero(m5[9])[0].tolist() == list(range(20))
    # W = 8 (two tiles, half-open interval): query at 5 (centre 6) takes centres in (2, 10] -> tiles 1, 2
    m2 = sta.axis_allowed(20, 4, 8)
    assert np.nonzero(m2[5])[0].tolist() == list(range(4, 12))
    # W = 4 (one tile): the query's own tile only
    m1 = sta.axis_allowed(20, 4, 4)
    assert np.nonzero(m1[13])[0].tolist() == [12, 13, 14, 15]


def test_mask_is_block_dense_and_symmetric():
    F, Hh, Ww = 8, 12, 16
    m = sta.sta_mask(F, Hh, Ww, window=(4, 12, 20))
    idx = np.arange(F * Hh * Ww).reshape(F, Hh, Ww)
    tiles = idx.reshape(F // 4, 4, Hh // 4, 4, Ww // 4, 4).transpose(0, 2, 4, 1, 3, 5).reshape(-1, 64)
    blocks = m[tiles[:, :, None, None], tiles[None, None, :, :]]      # [tq, 64, tk, 64]
    flat = blocks.transpose(0, 2, 1, 3).reshape(tiles.shape[0], tiles.shape[0], -1)
    assert np.all(flat.all(-1) | ~flat.any(-1))                        # each block all true or all false
    np.testing.assert_array_equal(m, m.T)                              # odd tile counts: symmetric


def test_three_tile_window_is_the_tile_neighbourhood():
    F, Hh, Ww, d = 8, 12, 16, 8
    q, k, v = _qkv(1, F * Hh * Ww, d)
    a = sta.sliding_tile_attention(q, k, v, F, Hh, Ww, window=(12, 12, 12))
    b = tile3d.local_attention(q, k, v, F, Hh, Ww, radius=1)
    np.testing.assert_allclose(a, b, rtol=1e-13, atol=1e-13)


def test_window_covering_the_grid_is_dense_attention():
    F, Hh, Ww, d = 4, 8, 12, 8
    q, k, v = _qkv(2, F * Hh * Ww, d)
    a = sta.sliding_tile_attention(q, k, v, F, Hh, Ww, window=(4, 12, 20))
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.tensor(q)[None, None], torch.tensor(k)[None, None], torch.tensor(v)[None, None])[0, 0].numpy()
    np.testing.assert_allclose(a, ref, rtol=0, atol=1e-12)


def test_single_queries_brute_force():
    F, Hh, Ww, d = 8, 16, 12, 4
    q, k, v = _qkv(3, F * Hh * Ww, d)
    window = (4, 20, 12)
    a = sta.sliding_tile_attention(q, k, v, F, Hh, Ww, window=window)
    idx = np.arange(F * Hh * Ww).reshape(F, Hh, Ww)

    def centre(x):
        return (x // 4) * 4 + 2

    for (f, h, w) in [(0, 0, 0), (7, 15, 11), (3, 9, 5), (4, 0, 11), (1, 7, 6)]:
        keys = [int(idx[x, y, z]) for x in range(F) for y in range(Hh) for z in range(Ww)
                if all(-W / 2 < centre(kk) - centre(qq) <= W / 2
                       for kk, qq, W in ((x, f, window[0]), (y, h, window[1]), (z, w, window[2])))]
        t = int(idx[f, h, w])
        lg = np.array([q[t] @ k[u] for u in keys]) / math.sqrt(d)
        p = np.exp(lg - lg.max())
        np.testing.assert_allclose(a[t], (p / p.sum()) @ v[keys], rtol=1e-12, atol=1e-13)


def test_rows_argument_computes_only_those_rows():
    F, Hh, Ww, d = 4, 8, 8, 4
    q, k, v = _qkv(4, F * Hh * Ww, d)
    full = sta.sliding_tile_attention(q, k, v, F, Hh, Ww, window=(4, 4, 12))
    part = sta.sliding_tile_attention(q, k, v, F, Hh, Ww, window=(4, 4, 12), rows=[0, 37, 255])
    np.testing.assert_allclose(part[[0, 37, 255]], full[[0, 37, 255]], rtol=1e-13, atol=1e-14)
    assert np.count_nonzero(part) == 3 * d
