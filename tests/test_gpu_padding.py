"""GPU parity on latents that are not a multiple of the tile (padded at the
high end of each axis to whole tiles; padding tokens are neither keys nor
queries), against the fp64 oracle.  Includes HunyuanVideo's own 720p latent
33 x 45 x 80 (the 5 s clip before any cropping), which no 6 x 8 x 8 tile
divides."""
import numpy as np
import pytest
import torch

import oracle
from parity_util import compare, compare_grad, dk_d_term, dq_d_term

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as s
    return s


def padded(latent, tile):
    return int(np.prod([-(-latent[i] // tile[i]) * tile[i] for i in range(3)]))


@pytest.mark.parametrize("latent,tile,row_shape,dtype", [
    ((13, 21, 18), (6, 8, 8), (128,), torch.bfloat16),
    ((33, 45, 80), (6, 8, 8), (64,), torch.bfloat16),
    ((13, 21, 18), (6, 8, 8), (), torch.float32),
    ((5, 7, 9), (2, 4, 4), (3,), torch.int16),
])
def test_padded_permutation(sta, latent, tile, row_shape, dtype):
    N = latent[0] * latent[1] * latent[2]
    Np = padded(latent, tile)
    g = torch.Generator().manual_seed(N)
    if dtype.is_floating_point:
        x = torch.randn((2, N) + row_shape, generator=g).to(dtype)
    else:
        x = torch.randint(-100, 100, (2, N) + row_shape, generator=g).to(dtype)
    xd = x.cuda()
    y = torch.full((2, Np) + row_shape, 7, dtype=dtype, device="cuda")
    sta.sta_tile_reorder(xd, y, latent, tile, token_dim=1)
    idx = torch.from_numpy(oracle.tile_major_index(latent, tile, np.arange(N)))
    expect = torch.zeros((2, Np) + row_shape, dtype=dtype)
    expect[:, idx] = x
    assert torch.equal(y.cpu(), expect)  # padding rows are zero
    z = torch.empty_like(xd)
    sta.sta_tile_unreorder(y, z, latent, tile, token_dim=1)
    assert torch.equal(z, xd)


def inputs(latent, B, H, d, seed):
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(seed)
    return [torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4)]


@pytest.mark.parametrize("latent,tile,B,H,d,windows", [
    ((13, 21, 18), (6, 8, 8), 1, 3, 128, [[6, 8, 8], [12, 16, 16], [18, 24, 24]]),
    ((9, 8, 20), (4, 8, 8), 2, 2, 64, [[8, 8, 16], [4, 8, 24]]),
    ((7, 9, 9), (2, 8, 8), 1, 2, 128, [[2, 8, 8], [8, 16, 16]]),
])
def test_padded_forward_and_backward_all_rows(sta, latent, tile, B, H, d, windows):
    check_all_rows(sta, latent, tile, B, H, d, windows)


def check_all_rows(sta, latent, tile, B, H, d, windows):
    """Forward and backward on every row against the oracle; the fused raster
    kernels (where the tile shape and latent allow them) equal the reorder chain."""
    q, k, v, do = inputs(latent, B, H, d, seed=sum(latent) * 7 + d)
    scale = 1.0 / np.sqrt(d)
    plan = sta.sta_plan(latent, tile, B, H, windows)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = sta.sta_attention(qd, kd, vd, plan, scale)
    o2, lse2 = sta.sta_attention(qd, kd, vd, plan, scale, fused=False)
    assert torch.equal(o, o2) and torch.equal(lse, lse2)  # fused raster path == reorder chain
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
            what=f"padded {latent}")
    dq, dk, dv = sta.sta_attention_backward(qd, kd, vd, o, lse, dod, plan, scale)
    chain = sta.sta_attention_backward(qd, kd, vd, o, lse, dod, plan, scale, fused=False)
    for a, b in zip((dq, dk, dv), chain):
        assert torch.equal(a, b)  # fused raster kernels == reorder, tile-major backward, unreorder
    assert sta.sta_last_device_status(plan) == 0
    rq, rk, rv = oracle.sta_backward(q, k, v, do, latent, tile, windows, scale)
    N = q.shape[2]
    bh = np.repeat(np.arange(B * H), N)
    pk_ref, _ = oracle.sta_attention(q, k, k, latent, tile, windows, scale)  # (P K) rows
    extra = {"dq": dq_d_term(o_ref.reshape(-1, d), pk_ref.reshape(-1, d), do.reshape(-1, d), scale),
             "dk": dk_d_term(q, k, v, o_ref, do, latent, tile, windows, scale).reshape(-1, d), "dv": None}
    for name, a, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        compare_grad(a.cpu().reshape(-1, d), r.reshape(-1, d), bh, what=f"{name} padded {latent}",
                     extra=extra[name])


@pytest.mark.parametrize("latent,tile,d", [
    ((6, 8, 8), (6, 8, 8), 128),    # the latent is exactly one tile
    ((5, 7, 8), (6, 8, 8), 64),     # smaller than one tile: a single padded tile
    ((1, 16, 16), (2, 8, 8), 128),  # the t axis is shorter than the tile
    ((3, 3, 40), (6, 8, 8), 128),   # one row of tiles along w, padded in t and h
])
def test_degenerate_latents_all_rows(sta, latent, tile, d):
    """Grids of one tile or one row of tiles, latents smaller than the tile:
    a one-tile window and a window three tiles wide on every axis (clamped to
    the volume)."""
    check_all_rows(sta, latent, tile, 1, 2, d, [list(tile), [3 * x for x in tile]])


def test_single_token_latent(sta):
    """A 1 x 1 x 1 latent: each row's softmax has one key, so O = V and
    dV = dO exactly (the weight is 1 and rounds to 1 in bf16), LSE is the one
    scaled score, and dQ, dK vanish up to fp32 rounding: dS = P (dO.v - dO.o)
    with o = v, the two dot products summed in different orders, at most
    d 2^-24 sum |dO_c v_c| (~6e-4 for these N(0, 1) rows) times scale |k| <= 0.5."""
    latent, tile, B, H, d = (1, 1, 1), (6, 8, 8), 2, 3, 128
    q, k, v, do = inputs(latent, B, H, d, seed=11)
    scale = 1.0 / np.sqrt(d)
    plan = sta.sta_plan(latent, tile, B, H, [list(tile)] * H)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = sta.sta_attention(qd, kd, vd, plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    assert torch.equal(o.cpu(), v)
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, [list(tile)] * H, scale)
    compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
            what="single token")
    dq, dk, dv = sta.sta_attention_backward(qd, kd, vd, o, lse, dod, plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    assert torch.equal(dv.cpu(), do)
    assert float(dq.abs().max()) <= 2.0 ** -10 and float(dk.abs().max()) <= 2.0 ** -10


def test_hunyuan_720p_latent_sampled(sta):
    """33 x 45 x 80 latent, tile 6 x 8 x 8 (padded to 36 x 48 x 80), window
    18 x 24 x 24, d = 128: sampled rows of corner and padded-edge tiles."""
    latent, tile, B, H, d = (33, 45, 80), (6, 8, 8), 1, 2, 128
    windows = [[18, 24, 24], [30, 40, 40]]
    q, k, v, _ = inputs(latent, B, H, d, seed=3345)
    plan = sta.sta_plan(latent, tile, B, H, windows)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, 1.0 / np.sqrt(d))
    assert sta.sta_last_device_status(plan) == 0
    n = [-(-latent[i] // tile[i]) for i in range(3)]
    tiles = [0, n[1] * n[2] - 1, (n[0] - 1) * n[1] * n[2], n[0] * n[1] * n[2] - 1,
             ((n[0] - 1) * n[1] + n[1] - 1) * n[2] + 4, (2 * n[1] + n[1] - 1) * n[2] + 3]
    rng = np.random.default_rng(5)
    toks = []
    for t in tiles:
        tt = oracle.tile_tokens(latent, tile, t)
        toks.extend(rng.choice(tt, min(24, len(tt)), replace=False).tolist() + [int(tt[0]), int(tt[-1])])
    toks = sorted(set(toks))
    rows = np.array([(h, t) for h in range(H) for t in toks], dtype=np.int64)
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, 1.0 / np.sqrt(d), rows=rows)
    og = o.reshape(-1, o.shape[2], d)[rows[:, 0], rows[:, 1]].cpu()
    lg = lse.reshape(-1, lse.shape[2])[rows[:, 0], rows[:, 1]].cpu()
    compare(og, lg, o_ref, lse_ref, what="33x45x80")


def test_padding_blocks_skipped_and_backward_ignores_their_rows(sta):
    """A block of padding rows only is not computed: tile-major O and LSE
    prefilled with NaN keep NaN there, every real row equals the raster
    forward, and the tile-major backward fed those very outputs (NaN rows
    included) gives the raster backward's bits: its row pass writes 0 for
    padding rows instead of reading them."""
    latent, tile, B, H, d = (9, 16, 16), (6, 8, 8), 1, 2, 128  # t: 9 = 6 + 3, so t 10-11 is one padding block
    windows = [[6, 8, 8], [12, 16, 16]]
    q, k, v, do = (x.cuda() for x in inputs(latent, B, H, d, seed=916))
    scale = 1.0 / np.sqrt(d)
    plan = sta.sta_plan(latent, tile, B, H, windows)
    Np = plan.padded_tokens
    qt, kt, vt, dot = (torch.empty((B, H, Np, d), dtype=torch.bfloat16, device="cuda") for _ in range(4))
    for x, y in ((q, qt), (k, kt), (v, vt), (do, dot)):
        sta.sta_tile_reorder(x, y, latent, tile)
    ot = torch.full((B, H, Np, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    lt = torch.full((B, H, Np), float("nan"), dtype=torch.float32, device="cuda")
    sta.sta_forward(plan, qt, kt, vt, ot, lt, scale)
    o, lse = sta.sta_attention(q, k, v, plan, scale)
    o_back, lse_back = torch.empty_like(o), torch.empty_like(lse)
    sta.sta_tile_unreorder(ot, o_back, latent, tile)
    sta.sta_tile_unreorder(lt, lse_back, latent, tile)
    assert torch.equal(o_back, o) and torch.equal(lse_back, lse)
    N = latent[0] * latent[1] * latent[2]
    real = set((oracle.tile_major_index(latent, tile, np.arange(N)) // 128).tolist())
    skipped = [b for b in range(Np // 128) if b not in real]
    assert skipped, "the geometry must have a block of padding rows only"
    for b in skipped:
        assert bool(torch.isnan(ot[:, :, 128 * b:128 * (b + 1)].float()).all())
        assert bool(torch.isnan(lt[:, :, 128 * b:128 * (b + 1)]).all())
    dq, dk, dv = sta.sta_backward(plan, qt, kt, vt, ot, lt, dot, scale)
    ref = sta.sta_attention_backward(q, k, v, o, lse, do, plan, scale)
    for x, r in zip((dq, dk, dv), ref):
        back = torch.empty_like(r)
        sta.sta_tile_unreorder(x, back, latent, tile)
        assert torch.equal(back, r)
    assert sta.sta_last_device_status(plan) == 0
