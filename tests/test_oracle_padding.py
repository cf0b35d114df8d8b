"""Pins of the oracle on latents that are not a multiple of the tile (padded
at the high end of each axis to whole tiles; windows placed on the padded
tile grid; padding tokens are neither keys nor queries).

- The token mask equals a brute-force mask built independently here: the
  tile grid of ceil(L / T) tiles per axis, the window as the in-range run of
  e tiles whose centre is nearest the query tile (ties low), keys = the real
  tokens of those tiles.
- Each row attends prod_d (min((s_d + e_d) T_d, L_d) - s_d T_d) keys.
- A window covering the padded grid gives dense softmax attention over the
  real tokens (scipy).
- Tile-major positions of the real tokens are distinct, inside the padded
  layout of n_tiles * |tile| rows, and follow raster order inside each tile.
"""
import itertools

import numpy as np
import pytest
import torch
from scipy.special import logsumexp, softmax

import oracle

CASES = [
    ((5, 7, 9), (2, 4, 4), [2, 4, 4]),
    ((5, 7, 9), (2, 4, 4), [4, 8, 8]),
    ((7, 6, 10), (3, 4, 4), [3, 4, 12]),
    ((4, 9, 5), (2, 2, 2), [2, 6, 2]),
    ((3, 3, 3), (2, 2, 2), [4, 2, 4]),
]


def ceil_div(a, b):
    return -(-a // b)


def nearest_run(q, e, n):
    best = None
    for s in range(0, n - e + 1):
        dist = abs((s + (e - 1) / 2.0) - q)
        if best is None or dist < best[0]:
            best = (dist, s)
    return best[1]


def brute_mask_padded(latent, tile, window):
    coords = np.array(list(itertools.product(*[range(x) for x in latent])))
    tiles = coords // np.array(tile)
    n = [ceil_div(latent[i], tile[i]) for i in range(3)]
    e = [min(window[i] // tile[i], n[i]) for i in range(3)]
    N = len(coords)
    mask = np.zeros((N, N), dtype=bool)
    for i in range(N):
        ok = np.ones(N, dtype=bool)
        for ax in range(3):
            s = nearest_run(int(tiles[i, ax]), e[ax], n[ax])
            ok &= (tiles[:, ax] >= s) & (tiles[:, ax] < s + e[ax])
        mask[i] = ok
    return mask, n, e


@pytest.mark.parametrize("latent,tile,window", CASES)
def test_mask_matches_brute_force_and_counts(latent, tile, window):
    mask, n, e = brute_mask_padded(latent, tile, window)
    N = mask.shape[0]
    coords = np.array(list(itertools.product(*[range(x) for x in latent])))
    for i in range(N):
        row = oracle.mask_row(latent, tile, window, i)
        assert np.array_equal(row, mask[i]), (latent, tile, window, i)
        count = 1
        for ax in range(3):
            s = nearest_run(int(coords[i, ax] // tile[ax]), e[ax], n[ax])
            count *= min((s + e[ax]) * tile[ax], latent[ax]) - s * tile[ax]
        assert row.sum() == count


def test_full_padded_window_is_dense():
    latent, tile, d = (5, 7, 9), (2, 4, 4), 8
    N = 5 * 7 * 9
    g = torch.Generator().manual_seed(21)
    q, k, v = (torch.randn(1, 1, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    win = [6, 8, 12]  # the padded grid 3 x 2 x 3 tiles
    o, lse = oracle.sta_attention(q, k, v, latent, tile, [win], 0.3)
    s = float(np.float32(0.3)) * (q[0, 0].double().numpy() @ k[0, 0].double().numpy().T)
    np.testing.assert_allclose(o[0, 0], softmax(s, axis=1) @ v[0, 0].double().numpy(), rtol=0, atol=1e-12)
    np.testing.assert_allclose(lse[0, 0], logsumexp(s, axis=1), rtol=0, atol=1e-12)


@pytest.mark.parametrize("latent,tile", [((5, 7, 9), (2, 4, 4)), ((33, 45, 80), (6, 8, 8))])
def test_padded_tile_major_positions(latent, tile):
    N = latent[0] * latent[1] * latent[2]
    n = [ceil_div(latent[i], tile[i]) for i in range(3)]
    vol = tile[0] * tile[1] * tile[2]
    pos = oracle.tile_major_index(latent, tile, np.arange(N))
    assert len(np.unique(pos)) == N
    assert pos.min() >= 0 and pos.max() < n[0] * n[1] * n[2] * vol
    # inside a tile, raster order of the tile's own offsets
    toks = oracle.tile_tokens(latent, tile, 0) if all(latent[i] >= tile[i] for i in range(3)) else None
    if toks is not None:
        assert np.array_equal(pos[toks], np.arange(vol))
    # the last tile of the padded grid holds the real tokens at the far corner
    t, h, w = latent[0] - 1, latent[1] - 1, latent[2] - 1
    last = (t * latent[1] + h) * latent[2] + w
    tile_id = ((t // tile[0]) * n[1] + h // tile[1]) * n[2] + w // tile[2]
    local = ((t % tile[0]) * tile[1] + h % tile[1]) * tile[2] + w % tile[2]
    assert pos[last] == tile_id * vol + local
