"""CPU emulation of the forward kernel's key-split arithmetic against the oracle.

The forward kernel splits every 128-key chunk of a query block's key list
between two softmax halves (keys 0-63 and 64-127 of the chunk).  The two warps
that own the same 32 rows keep one running maximum m per row and one fp32
output accumulator O between them; each half keeps its own row sum.  The
block's first chunk sets m to the maximum of both halves' scores (a stand-in 0
when that chunk holds padding keys only); later chunks are exponentiated
against m, and when any row of the 32-row group has a half-row sum above
65536 the group raises m to the maximum of m and both halves' chunk maxima,
rescaling O and both row sums (the slow path).  P is rounded to bf16 before
P V, and the row sums add those rounded values.  The epilogue writes
O / (l_A + l_B) in bf16 and LSE = m scale + ln(l_A + l_B).

This file restates those steps in numpy, in the kernel's order and
precisions, and checks them against the fp64 oracle with the tolerances of
the GPU parity tests.  It pins the algorithm, not the CUDA code: cases cover a
divisible latent, a padded one, a latent whose second halves never hold a
real key (one t-slice), and inputs that force the rescale (at the largest
factor the exponentials would overflow fp32 without it).  Planting a missing
rescale of O, a row sum of only one half, or unmasked padding keys here fails
some of its cases.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sparse_attention_video_sta_b200 as sta
from parity_util import LSE_REL_TOL, O_MEAN_TOL, o_bound

LOG2E = 1.4426950408889634
RESCALE_ROW_SUM = 65536.0


def bf16(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).to(torch.float32).numpy()


def tile_major_tokens(latent, tile, tile_id):
    """Raster token of each tile-major row of a tile (-1 for padding rows)."""
    n = [-(-latent[i] // tile[i]) for i in range(3)]
    it, rem = divmod(tile_id, n[1] * n[2])
    ih, iw = divmod(rem, n[2])
    out = []
    for lt in range(tile[0]):
        for lh in range(tile[1]):
            for lw in range(tile[2]):
                t, h, w = it * tile[0] + lt, ih * tile[1] + lh, iw * tile[2] + lw
                real = t < latent[0] and h < latent[1] and w < latent[2]
                out.append((t * latent[1] + h) * latent[2] + w if real else -1)
    return np.array(out, dtype=np.int64)


def emulate_block(qr, k, v, key_tiles, latent, tile, scale):
    """One 128-row query block: qr [128, d] fp32; k, v [N, d] fp32 (raster).
    Returns O [128, d] (bf16 values) and LSE [128]."""
    c = np.float32(scale * LOG2E)
    d = qr.shape[1]
    m = np.zeros(128, np.float32)
    lh = [np.zeros(128, np.float32), np.zeros(128, np.float32)]
    o = np.zeros((128, d), np.float32)
    first = True
    for kt in key_tiles:
        toks = tile_major_tokens(latent, tile, kt)
        for ch in range(len(toks) // 128):
            s_h, v_h = [], []
            for h in range(2):
                keys = toks[ch * 128 + 64 * h: ch * 128 + 64 * h + 64]
                real = keys >= 0
                kk = np.where(real[:, None], k[np.maximum(keys, 0)], 0.0).astype(np.float32)
                v_h.append(np.where(real[:, None], v[np.maximum(keys, 0)], 0.0).astype(np.float32))
                s = (qr.astype(np.float64) @ kk.astype(np.float64).T).astype(np.float32)
                s[:, ~real] = -np.inf
                s_h.append(s)
            mx = np.maximum(s_h[0].max(axis=1), s_h[1].max(axis=1))
            alpha = np.ones(128, np.float32)
            if first:
                m = np.where(mx == -np.inf, 0.0, mx).astype(np.float32)
            else:
                with np.errstate(over="ignore"):  # inf here is caught by the row-sum test
                    sums = [bf16(np.exp2(s * c - m[:, None] * c)).sum(axis=1, dtype=np.float32) for s in s_h]
                need = ~(sums[0] <= RESCALE_ROW_SUM) | ~(sums[1] <= RESCALE_ROW_SUM)
                slow = np.repeat(need.reshape(4, 32).any(axis=1), 32)  # per 32-row warp pair
                grow = slow & ((mx - m) * c > 0)
                alpha = np.exp2(np.where(grow, (m - mx) * c, 0.0)).astype(np.float32)
                m = np.where(grow, mx, m).astype(np.float32)
            o = o * alpha[:, None]
            for h in range(2):
                p = bf16(np.exp2(s_h[h] * c - m[:, None] * c).astype(np.float32))
                lh[h] = lh[h] * alpha + p.sum(axis=1, dtype=np.float32)
                o = o + p @ bf16(v_h[h])
            if first:
                first = False
    lsum = lh[0] + lh[1]
    out = (o * (np.float32(1.0) / lsum)[:, None]).astype(np.float32)
    lse = m * np.float32(scale) + np.log(lsum)
    return bf16(out), lse


def run_case(latent, tile, windows, d, k_boost=None, seed=0):
    H = len(windows)
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(1, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    if k_boost is not None:  # a few late keys with large scores force the lazy rescale
        toks, f = k_boost
        k[:, :, toks] = (k[:, :, toks].float() * f).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    plan = sta.sta_plan_host(latent, tile, 1, H, windows)
    qf, kf, vf = (x.float().numpy() for x in (q, k, v))
    n_tiles = plan.tiles_per_head
    got_o = np.full((H, N, d), np.nan)
    got_l = np.full((H, N), np.nan)
    for h in range(H):
        for t in range(n_tiles):
            toks = tile_major_tokens(latent, tile, t)
            key_tiles = plan.query(h, t)
            for blk in range(len(toks) // 128):
                rows = toks[blk * 128: blk * 128 + 128]
                if not (rows >= 0).any():
                    continue  # blocks of padding rows only are not computed
                qr = np.where((rows >= 0)[:, None], qf[0, h, np.maximum(rows, 0)], 0.0).astype(np.float32)
                o, lse = emulate_block(qr, kf[0, h], vf[0, h], key_tiles, latent, tile, scale)
                got_o[h, rows[rows >= 0]] = o[rows >= 0]
                got_l[h, rows[rows >= 0]] = lse[rows >= 0]
    ref_o, ref_l = o_ref[0], lse_ref[0]
    assert not np.isnan(got_o).any() and not np.isnan(got_l).any()
    do = np.abs(got_o - ref_o)
    assert (do <= o_bound(ref_o)).all(), float(do.max())
    assert do.mean() <= O_MEAN_TOL
    dl = np.abs(got_l - ref_l) / np.maximum(np.abs(ref_l), 1.0)
    assert dl.max() <= LSE_REL_TOL, float(dl.max())


def test_divisible_latent():
    run_case((12, 16, 16), (6, 8, 8), [(6, 8, 8), (12, 16, 16)], 64)


def test_padded_latent():
    run_case((7, 9, 10), (6, 8, 8), [(6, 8, 8), (12, 16, 16)], 64, seed=1)


def test_half_without_real_keys():
    # One t-slice: in every chunk the second half (tile offset t = 1) is padding.
    run_case((1, 8, 8), (6, 8, 8), [(6, 8, 8)], 64, seed=2)
    run_case((1, 12, 13), (6, 8, 8), [(6, 16, 16), (6, 8, 8)], 32, seed=3)


@pytest.mark.parametrize("factor", [4.0, 12.0, 40.0])
def test_lazy_rescale(factor):
    # Keys of the last tile (visited last by every query tile whose window
    # holds it) get large scores, so their chunks exceed the row-sum bound;
    # at the largest factor, exponentials against the first chunk's maximum
    # would overflow fp32 without the rescale.
    latent, tile = (12, 16, 16), (6, 8, 8)
    last = tile_major_tokens(latent, tile, 7)
    run_case(latent, tile, [(12, 16, 16)], 64, k_boost=(torch.from_numpy(last[::7]), factor), seed=4)
