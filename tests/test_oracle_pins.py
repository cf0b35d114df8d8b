"""Pins of the CPU oracle against facts other than itself.

Each test fixes the oracle to something independent of its own code: a figure
printed on the pages (tests/golden), a closed form computed with a library
routine (dense attention via numpy matmul + scipy logsumexp), brute force with
a different algorithm (window chosen by enumerating every in-range start and
taking the nearest centre), or an invariant of softmax attention.  A dropped
scale, a wrong sign or index, swapped operands, a truncated instead of shifted
window, a log2 LSE or a wrong token order each fail at least one test here.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch
from scipy.special import logsumexp

import oracle
import sta_inputs

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------
# Independent helpers (brute force, library routines)
# --------------------------------------------------------------------------

def nearest_centre_window(q: int, e: int, n: int) -> range:
    """Among all in-range windows [s, s+e) of an axis of n tiles, the one whose
    centre is nearest to tile q; ties go to the lower start."""
    best = None
    for s in range(0, n - e + 1):
        dist = abs((s + (e - 1) / 2.0) - q)
        if best is None or dist < best[0]:
            best = (dist, s)
    return range(best[1], best[1] + e)


def brute_mask(latent, tile, window) -> np.ndarray:
    """N x N token mask built tile set by tile set with the nearest-centre rule."""
    N = latent[0] * latent[1] * latent[2]
    coords = np.array(list(itertools.product(*[range(x) for x in latent])))  # raster
    tiles = coords // np.array(tile)
    n = [latent[i] // tile[i] for i in range(3)]
    e = [min(window[i] // tile[i], n[i]) for i in range(3)]
    mask = np.zeros((N, N), dtype=bool)
    for i in range(N):
        ok = np.ones(N, dtype=bool)
        for ax in range(3):
            win = nearest_centre_window(int(tiles[i, ax]), e[ax], n[ax])
            ok &= (tiles[:, ax] >= win.start) & (tiles[:, ax] < win.stop)
        mask[i] = ok
    return mask


def bf16_to_f64(x: torch.Tensor) -> np.ndarray:
    return x.to(torch.float64).numpy()


def dense_masked_attention(q, k, v, mask, scale):
    """Masked softmax attention with numpy matmul and scipy logsumexp (fp64).
    q, k, v: [N, d] float64; mask: [N, N] bool."""
    s = scale * (q @ k.T)
    s = np.where(mask, s, -np.inf)
    lse = logsumexp(s, axis=1)
    p = np.exp(s - lse[:, None])
    return p @ v, lse


def rand_bf16(shape, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randn(*shape, generator=g).to(torch.bfloat16)


# --------------------------------------------------------------------------
# Mask / window pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("n", range(1, 10))
def test_window_start_matches_nearest_centre_enumeration(n):
    # One axis of n tiles (tile = 1 token): the oracle's key set for every query
    # and every window extent (including windows wider than the axis) must be
    # the nearest-centre in-range window.
    latent, tile = (n, 1, 1), (1, 1, 1)
    for w in range(1, n + 3):
        e = min(w, n)
        for q in range(n):
            row = oracle.mask_row(latent, tile, (w, 1, 1), q)
            got = set(np.nonzero(row)[0].tolist())
            assert got == set(nearest_centre_window(q, e, n)), (n, w, q)


def test_mask_matches_brute_force_3d():
    rng = np.random.default_rng(7)
    cases = [((5, 6, 7), (1, 1, 1)), ((4, 6, 8), (2, 2, 2)), ((6, 4, 6), (3, 2, 1)),
             ((2, 3, 4), (1, 1, 1))]
    for latent, tile in cases:
        n = [latent[i] // tile[i] for i in range(3)]
        for _ in range(6):
            window = tuple(int(rng.integers(1, n[i] + 2)) * tile[i] for i in range(3))
            bm = brute_mask(latent, tile, window)
            N = bm.shape[0]
            for qi in range(N):
                assert np.array_equal(oracle.mask_row(latent, tile, window, qi), bm[qi]), \
                    (latent, tile, window, qi)


def test_no_mixed_blocks_and_tile_shared_rows():
    # Every (query tile, key tile) block is fully attended or fully skipped, and
    # all queries of one tile share one key set.
    latent, tile = (4, 6, 8), (2, 2, 2)
    for window in [(2, 2, 2), (4, 4, 4), (2, 6, 4), (4, 6, 8), (8, 8, 8)]:
        bm = np.stack([oracle.mask_row(latent, tile, window, i) for i in range(4 * 6 * 8)])
        n_tiles = (latent[0] // tile[0]) * (latent[1] // tile[1]) * (latent[2] // tile[2])
        toks = [oracle.tile_tokens(latent, tile, t) for t in range(n_tiles)]
        for a in range(n_tiles):
            for b in range(n_tiles):
                blk = bm[np.ix_(toks[a], toks[b])]
                assert blk.all() or not blk.any(), (window, a, b)
            rows = bm[toks[a]]
            assert (rows == rows[0]).all()


@pytest.mark.parametrize("latent,tile,window", [
    ((18, 24, 24), (6, 8, 8), (12, 16, 16)),
    ((30, 48, 80), (6, 8, 8), (30, 40, 40)),
    ((30, 48, 80), (6, 8, 8), (60, 96, 160)),
    ((12, 16, 24), (6, 8, 8), (6, 8, 8)),
])
def test_attended_tiles_equal_clamped_window_volume(latent, tile, window):
    n = [latent[i] // tile[i] for i in range(3)]
    e = [min(window[i] // tile[i], n[i]) for i in range(3)]
    vol = tile[0] * tile[1] * tile[2]
    rng = np.random.default_rng(3)
    N = oracle.num_tokens(latent)
    for qi in rng.integers(0, N, size=12).tolist() + [0, N - 1]:
        row = oracle.mask_row(latent, tile, window, qi)
        assert row.sum() == e[0] * e[1] * e[2] * vol
        assert row[qi]  # a query always sees its own tile


def test_pages_sparsity_pin_720p():
    """The pages report 91% sparsity for w=(18,24,24) on the 720p 5 s latent."""
    with open(os.path.join(GOLDEN, "sparsity_720p_w18x24x24.json")) as f:
        gold = json.load(f)
    latent, tile, window = tuple(gold["latent"]), tuple(gold["tile"]), tuple(gold["window"])
    N = oracle.num_tokens(latent)
    n_tiles = N // (tile[0] * tile[1] * tile[2])
    allowed = 0
    for t in range(n_tiles):
        toks = oracle.tile_tokens(latent, tile, t)
        row = oracle.mask_row(latent, tile, window, int(toks[0]))
        allowed += int(row.sum()) * len(toks)
        if t % 37 == 0:  # rows inside one tile are identical
            assert np.array_equal(oracle.mask_row(latent, tile, window, int(toks[-1])), row)
    sparsity = 1.0 - allowed / float(N) / float(N)
    assert abs(sparsity - gold["value"]) <= gold["printed_precision"]
    assert math.isclose(sparsity, 1.0 - 27.0 / 300.0, rel_tol=0, abs_tol=1e-12)


# --------------------------------------------------------------------------
# Attention value pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("window", [(12, 16, 16), (60, 96, 160)])
def test_full_window_equals_dense_attention(window):
    latent, tile, d = (12, 16, 16), (6, 8, 8), 16
    N = oracle.num_tokens(latent)
    q, k, v = (rand_bf16((1, 1, N, d), s) for s in (11, 12, 13))
    scale = 1.0 / math.sqrt(d)
    O, lse = oracle.sta_attention(q, k, v, latent, tile, [window], scale)
    qd, kd, vd = (bf16_to_f64(x[0, 0]) for x in (q, k, v))
    O_ref, lse_ref = dense_masked_attention(qd, kd, vd, np.ones((N, N), bool),
                                            float(np.float32(scale)))
    assert np.max(np.abs(O[0, 0] - O_ref)) <= 1e-12
    assert np.max(np.abs(lse[0, 0] - lse_ref)) <= 1e-12


def test_single_tile_window_is_block_diagonal():
    latent, tile, d = (12, 16, 16), (6, 8, 8), 8
    N = oracle.num_tokens(latent)
    q, k, v = (rand_bf16((1, 1, N, d), s) for s in (21, 22, 23))
    scale = 0.37
    O, lse = oracle.sta_attention(q, k, v, latent, tile, [tile], scale)
    qd, kd, vd = (bf16_to_f64(x[0, 0]) for x in (q, k, v))
    for t in range(8):
        toks = oracle.tile_tokens(latent, tile, t)
        n = len(toks)
        O_ref, lse_ref = dense_masked_attention(qd[toks], kd[toks], vd[toks],
                                                np.ones((n, n), bool), float(np.float32(scale)))
        assert np.max(np.abs(O[0, 0, toks] - O_ref)) <= 1e-12
        assert np.max(np.abs(lse[0, 0, toks] - lse_ref)) <= 1e-12


@pytest.mark.parametrize("latent,tile,windows", [
    ((2, 3, 4), (1, 1, 1), [(1, 3, 3), (2, 2, 3)]),      # 3D neighbourhood attention
    ((4, 6, 8), (2, 2, 2), [(2, 4, 4), (4, 2, 6)]),
    ((6, 4, 6), (3, 2, 1), [(3, 2, 3), (6, 4, 2)]),
])
def test_brute_force_tiny_volumes(latent, tile, windows):
    N = oracle.num_tokens(latent)
    d, B, H = 8, 2, len(windows)
    q, k, v = (rand_bf16((B, H, N, d), s) for s in (31, 32, 33))
    scale = 0.6
    O, lse = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    for b in range(B):
        for h in range(H):
            m = brute_mask(latent, tile, windows[h])
            qd, kd, vd = (bf16_to_f64(x[b, h]) for x in (q, k, v))
            O_ref, lse_ref = dense_masked_attention(qd, kd, vd, m, float(np.float32(scale)))
            assert np.max(np.abs(O[b, h] - O_ref)) <= 1e-12
            assert np.max(np.abs(lse[b, h] - lse_ref)) <= 1e-12


def test_invariants_rows_sum_to_one_hull_and_lse():
    latent, tile, d = (12, 16, 16), (6, 8, 8), 16
    N = oracle.num_tokens(latent)
    window = (6, 16, 8)
    q, k = rand_bf16((1, 1, N, d), 41), rand_bf16((1, 1, N, d), 42)
    ones = torch.ones((1, 1, N, d), dtype=torch.bfloat16)
    scale = 0.25
    # softmax weights sum to one: with V = 1 every output is exactly 1
    O1, _ = oracle.sta_attention(q, k, ones, latent, tile, [window], scale)
    assert np.max(np.abs(O1 - 1.0)) <= 1e-13
    # O lies in the per-coordinate hull of the attended values; exp(LSE) is the
    # sum of exp(scores) over attended keys
    v = rand_bf16((1, 1, N, d), 43)
    O, lse = oracle.sta_attention(q, k, v, latent, tile, [window], scale)
    qd, kd, vd = (bf16_to_f64(x[0, 0]) for x in (q, k, v))
    for qi in [0, 17, 555, N - 1]:
        row = oracle.mask_row(latent, tile, window, qi)
        lo, hi = vd[row].min(axis=0), vd[row].max(axis=0)
        assert np.all(O[0, 0, qi] >= lo - 1e-12) and np.all(O[0, 0, qi] <= hi + 1e-12)
        s = float(np.float32(scale)) * (kd[row] @ qd[qi])
        assert abs(math.exp(lse[0, 0, qi] - s.max()) - np.exp(s - s.max()).sum()) <= 1e-9 * row.sum()


def test_row_subset_matches_full_evaluation():
    # The sampled-row interface (used at large sizes) returns the same numbers
    # as the whole-volume evaluation.
    latent, tile, d = (12, 16, 16), (6, 8, 8), 16
    N = oracle.num_tokens(latent)
    q, k, v = (rand_bf16((2, 2, N, d), s) for s in (51, 52, 53))
    wins = [(6, 8, 8), (12, 16, 8)]
    O, lse = oracle.sta_attention(q, k, v, latent, tile, wins, 0.3)
    rows = np.array([[0, 5], [3, 1000], [2, N - 1], [1, 77]], dtype=np.int64)
    Os, lses = oracle.sta_attention(q, k, v, latent, tile, wins, 0.3, rows=rows)
    for i, (bh, t) in enumerate(rows):
        assert np.array_equal(Os[i], O[bh // 2, bh % 2, t])
        assert lses[i] == lse[bh // 2, bh % 2, t]


# --------------------------------------------------------------------------
# Token permutation pins
# --------------------------------------------------------------------------

@pytest.mark.parametrize("latent,tile", [((18, 24, 24), (6, 8, 8)), ((4, 6, 8), (2, 3, 2)),
                                         ((12, 16, 24), (6, 8, 8))])
def test_tile_major_order_is_a_bijection_of_contiguous_cubes(latent, tile):
    N = oracle.num_tokens(latent)
    idx = oracle.tile_major_index(latent, tile, np.arange(N))
    assert np.array_equal(np.sort(idx), np.arange(N))
    vol = tile[0] * tile[1] * tile[2]
    coords = np.array(list(itertools.product(*[range(x) for x in latent])))
    inv = np.empty(N, dtype=np.int64)
    inv[idx] = np.arange(N)
    n = [latent[i] // tile[i] for i in range(3)]
    for t in range(N // vol):
        toks = inv[t * vol:(t + 1) * vol]
        c = coords[toks]
        # one cube per tile, tiles in raster order over the tile grid
        it, ih, iw = np.unravel_index(t, n)
        assert (c[:, 0] // tile[0] == it).all() and (c[:, 1] // tile[1] == ih).all() \
            and (c[:, 2] // tile[2] == iw).all()
        # tokens inside a tile in raster order
        assert np.all(np.diff(toks) > 0)


# --------------------------------------------------------------------------
# Input generator checks
# --------------------------------------------------------------------------

def test_inputs_are_seeded_and_shaped():
    w = sta_inputs.WORKLOADS[1]
    a = sta_inputs.make_slice(w, 0, 0, 1)
    b = sta_inputs.make_slice(w, 0, 0, 1)
    c = sta_inputs.make_slice(w, 1, 0, 1)
    assert a.dtype == torch.bfloat16 and a.shape == (w.tokens, w.head_dim)
    assert torch.equal(a, b) and not torch.equal(a, c)
    w3 = sta_inputs.WORKLOADS[3]
    wins = sta_inputs.windows(w3)
    assert wins.shape == (24, 3)
    assert set(map(tuple, wins.tolist())) <= set(sta_inputs.MIXED_CHOICES)
    assert torch.equal(wins, sta_inputs.windows(w3))
    f = sta_inputs.head_factors(sta_inputs.WORKLOADS[5])
    assert f.shape == (24,) and float(f.min()) >= 0.5 and float(f.max()) <= 2.0
