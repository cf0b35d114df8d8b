"""GPU parity: the CUDA path (through the C ABI) against the fp64 CPU oracle.

Every test here needs a B200 (sm_100a).  Inputs come from the seeded generator
module ``sta_inputs``; expected values come only from ``oracle``.
"""
import math

import numpy as np
import pytest
import torch

import oracle
import sta_inputs
from parity_util import compare, oracle_rows, sample_tiles, tile_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as s
    return s


def gather_rows(o, lse, rows, H):
    bh = torch.from_numpy(rows[:, 0])
    tok = torch.from_numpy(rows[:, 1])
    o_c = o.reshape(-1, o.shape[2], o.shape[3])
    l_c = lse.reshape(-1, lse.shape[2])
    idx_bh, idx_t = bh.to(o.device), tok.to(o.device)
    return o_c[idx_bh, idx_t].cpu(), l_c[idx_bh, idx_t].cpu()


# ---------------------------------------------------------------- permutation

@pytest.mark.parametrize("latent,tile,outer,row_shape,dtype", [
    ((18, 24, 24), (6, 8, 8), 2, (64,), torch.bfloat16),
    ((30, 48, 80), (6, 8, 8), 3, (128,), torch.bfloat16),
    ((30, 48, 80), (6, 8, 8), 4, (), torch.float32),        # LSE rows, 4 bytes
    ((12, 16, 16), (4, 8, 8), 1, (3,), torch.int16),         # 6-byte rows
    ((6, 8, 16), (2, 4, 8), 5, (1,), torch.uint8),           # 1-byte rows
])
def test_permutation_bit_exact(sta, latent, tile, outer, row_shape, dtype):
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator(device="cpu").manual_seed(N + outer)
    if dtype.is_floating_point:
        x = torch.randn((outer, N) + row_shape, generator=g).to(dtype)
    else:
        x = torch.randint(-100, 100, (outer, N) + row_shape, generator=g).to(dtype)
    xd = x.cuda()
    y = torch.empty_like(xd)
    sta.sta_tile_reorder(xd, y, latent, tile, token_dim=1)
    idx = torch.from_numpy(oracle.tile_major_index(latent, tile, np.arange(N)))
    expect = torch.empty_like(x)
    expect[:, idx] = x
    assert torch.equal(y.cpu(), expect)
    z = torch.empty_like(xd)
    sta.sta_tile_unreorder(y, z, latent, tile, token_dim=1)
    assert torch.equal(z, xd)


# ---------------------------------------------------------------- forward

def run_full_oracle(sta, latent, tile, B, H, d, windows, scale, seed):
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(seed)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    plan = sta.sta_plan(latent, tile, B, H, windows)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    return compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d),
                   lse_ref.reshape(-1), what=f"{latent} {tile} {windows}")


def test_forward_tiny_workload_all_rows(sta):
    w = sta_inputs.WORKLOADS[1]
    q, k, v = sta_inputs.make_qkv(w)
    wins = sta_inputs.windows(w).tolist()
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, wins)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, w.softmax_scale)
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, w.latent, w.tile, wins, w.softmax_scale)
    compare(o.cpu().reshape(-1, w.head_dim), lse.cpu().reshape(-1),
            o_ref.reshape(-1, w.head_dim), lse_ref.reshape(-1), what="tiny")


@pytest.mark.parametrize("latent,tile,B,H,d,windows", [
    ((12, 16, 16), (6, 8, 8), 1, 2, 128, [(6, 8, 8), (12, 16, 16)]),       # 1 tile / full window
    ((12, 16, 16), (4, 8, 8), 2, 3, 64, [(4, 8, 8), (8, 16, 8), (12, 16, 16)]),   # 256-token tiles
    ((6, 16, 32), (2, 8, 8), 1, 2, 128, [(2, 8, 8), (6, 16, 16)]),           # 128-token tiles
    ((18, 24, 16), (6, 8, 8), 2, 1, 64, [(30, 48, 48)]),                     # window > volume
    ((12, 24, 24), (6, 8, 8), 1, 2, 128, [(6, 16, 8), (12, 8, 24)]),         # even windows
])
def test_forward_small_geometries_all_rows(sta, latent, tile, B, H, d, windows):
    run_full_oracle(sta, latent, tile, B, H, d, windows, 1.0 / math.sqrt(d), seed=d + H)


def sampled_parity(sta, idx, heads, n_random, rows_per_tile, fused=True):
    w = sta_inputs.WORKLOADS[idx]
    wins = sta_inputs.windows(w).tolist()
    q, k, v = sta_inputs.make_qkv(w, heads=heads)
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, wins)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, w.softmax_scale, fused=fused)
    assert sta.sta_last_device_status(plan) == 0
    tiles = sample_tiles(w.latent, w.tile, n_random, seed=idx)
    toks = tile_rows(w.latent, w.tile, tiles, rows_per_tile, seed=idx)
    bhs = [b * w.heads + h for b in range(w.batch) for h in heads]
    rows, o_ref, lse_ref = oracle_rows(q, k, v, w.latent, w.tile, wins, w.softmax_scale, bhs, toks)
    og, lg = gather_rows(o, lse, rows, w.heads)
    stats = compare(og, lg, o_ref, lse_ref, what=f"workload {idx}" + ("" if fused else " (permuted path)"))
    return w, plan, o, lse, stats


@pytest.mark.parametrize("fused", [True, False])
def test_forward_720p_sampled(sta, fused):
    w, plan, o, lse, _ = sampled_parity(sta, 2, heads=[0, 7, 16, 23], n_random=3, rows_per_tile=None,
                                        fused=fused)
    # heads that were not drawn hold zeros: every score is 0, so O = 0 exactly
    # and LSE = ln(27 * 384) (27 key tiles of 384 tokens)
    zero = [h for h in range(w.heads) if h not in (0, 7, 16, 23)]
    oz = o[:, zero]
    assert torch.count_nonzero(oz).item() == 0
    lz = lse[:, zero].double().cpu()
    assert float((lz - math.log(27 * 384)).abs().max()) <= 1e-5


def test_forward_mixed_windows_sampled(sta):
    w = sta_inputs.WORKLOADS[3]
    wins = sta_inputs.windows(w).tolist()
    heads = []
    for choice in sta_inputs.MIXED_CHOICES:
        hs = [h for h, x in enumerate(wins) if tuple(x) == choice]
        heads += hs[:2]
    sampled_parity(sta, 3, heads=heads, n_random=2, rows_per_tile=64)


def test_forward_full_window_sampled(sta):
    sampled_parity(sta, 4, heads=[3, 20], n_random=3, rows_per_tile=48)


def test_forward_large_scaled_sampled(sta):
    # batch 2, per-head scale factors in [0.5, 2]
    sampled_parity(sta, 5, heads=[1, 13], n_random=3, rows_per_tile=48)


# ---------------------------------------------------------------- behaviour

def test_forward_is_deterministic_and_stream_ordered(sta):
    w = sta_inputs.WORKLOADS[1]
    q, k, v = (t.cuda() for t in sta_inputs.make_qkv(w))
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    s = torch.cuda.Stream()
    with torch.cuda.stream(s):
        o1, l1 = sta.sta_attention(q, k, v, plan, w.softmax_scale)
        o2, l2 = sta.sta_attention(q, k, v, plan, w.softmax_scale)
    s.synchronize()
    assert torch.equal(o1, o2) and torch.equal(l1, l2)
    assert sta.sta_last_device_status(plan, s) == 0


def test_device_timeout_is_reported_and_context_survives(sta):
    w = sta_inputs.WORKLOADS[1]
    q, k, v = (t.cuda() for t in sta_inputs.make_qkv(w))
    plan = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    o_ok, l_ok = sta.sta_attention(q, k, v, plan, w.softmax_scale)
    assert sta.sta_last_device_status(plan) == 0
    sta.sta_debug_inject_timeout(True, 30)
    try:
        sta.sta_attention(q, k, v, plan, w.softmax_scale)
        assert sta.sta_last_device_status(plan) == sta.STA_ERR_TIMEOUT
    finally:
        sta.sta_debug_inject_timeout(False, 30)
    # the status was cleared and the context still works
    o2, l2 = sta.sta_attention(q, k, v, plan, w.softmax_scale)
    assert sta.sta_last_device_status(plan) == 0
    assert torch.equal(o2, o_ok) and torch.equal(l2, l_ok)


def test_timeout_with_copies_in_flight_is_reported_and_next_call_is_clean(sta):
    """A wait runs out at each CTA's second work item, after the first item
    was computed and the second item's query block and K/V chunks were issued:
    the kernel drains those copies and its MMAs and exits.  The status is
    TIMEOUT, and the next call gives the same bits as a clean one."""
    latent, tile, B, H, d = (30, 48, 80), (6, 8, 8), 1, 2, 128
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator(device="cuda").manual_seed(909)
    q, k, v = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    plan = sta.sta_plan(latent, tile, B, H, [(18, 24, 24), (30, 40, 40)])
    assert plan.stats()[1] >= 2 * 148  # every CTA takes a second item
    for fused in (True, False):
        o_ok, l_ok = sta.sta_attention(q, k, v, plan, fused=fused)
        assert sta.sta_last_device_status(plan) == 0
        sta.sta_debug_inject_timeout(2, 30)
        try:
            sta.sta_attention(q, k, v, plan, fused=fused)
            assert sta.sta_last_device_status(plan) == sta.STA_ERR_TIMEOUT
        finally:
            sta.sta_debug_inject_timeout(0, 30)
        o2, l2 = sta.sta_attention(q, k, v, plan, fused=fused)
        assert sta.sta_last_device_status(plan) == 0
        assert torch.equal(o2, o_ok) and torch.equal(l2, l_ok)


def test_shape_mismatch_rejected_before_launch(sta):
    plan = sta.sta_plan((18, 24, 24), (6, 8, 8), 1, 2, [(12, 16, 16)] * 2)
    q = torch.zeros(1, 2, 10368, 64, dtype=torch.bfloat16, device="cuda")
    bad = torch.zeros(1, 3, 10368, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 2, 10368, dtype=torch.float32, device="cuda")
    with pytest.raises(ValueError):
        sta.sta_forward(plan, q, bad, q, q, lse, 0.125)
    with pytest.raises(sta.StaError):
        sta.sta_forward(plan, q, q, q, torch.empty_like(q), lse, -1.0)
    q96 = torch.zeros(1, 2, 10368, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sta.StaError) as e:
        sta.sta_forward(plan, q96, q96, q96, torch.empty_like(q96), lse, 0.1)
    assert e.value.status == sta.STA_ERR_UNSUPPORTED


# ---------------------------------------------------------------- online-softmax rescale paths

def test_forward_running_max_grows_every_chunk(sta):
    # Scores rise by 12 log2-units from one 32-key chunk (in the kernel's visit
    # order: ascending tile id, tile-major inside a tile) to the next, so the
    # running max moves inside every row step and across steps: the P already
    # written, the row sum and O are all rescaled many times.
    latent, tile, d = (6, 16, 16), (6, 8, 8), 64
    N = latent[0] * latent[1] * latent[2]
    scale = 1.0 / math.sqrt(d)
    c = scale * 1.4426950408889634
    tm = oracle.tile_major_index(latent, tile, np.arange(N))   # visit position of each raster key
    q = torch.zeros(1, 1, N, d)
    q[..., 0] = 8.0
    k = torch.zeros(1, 1, N, d)
    k[0, 0, :, 0] = torch.from_numpy(12.0 * (tm // 32) / (c * 8.0)).float()
    g = torch.Generator().manual_seed(5)
    v = torch.randn(1, 1, N, d, generator=g)
    q, k, v = (t.to(torch.bfloat16) for t in (q, k, v))
    windows = [latent]
    plan = sta.sta_plan(latent, tile, 1, 1, windows)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
            what="rising max")


@pytest.mark.parametrize("factor", [4.0, 6.0])
def test_forward_sharp_softmax_random(sta, factor):
    # Q and K scaled so logits have std ~factor^2: row maxima jump by far more
    # than 2^8 between chunks early in a row.
    latent, tile, B, H, d = (12, 16, 16), (6, 8, 8), 1, 2, 128
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(int(factor * 10))
    q, k = ((factor * torch.randn(B, H, N, d, generator=g)).to(torch.bfloat16) for _ in range(2))
    v = torch.randn(B, H, N, d, generator=g).to(torch.bfloat16)
    windows = [(12, 16, 8), (12, 16, 16)]
    scale = 1.0 / math.sqrt(d)
    plan = sta.sta_plan(latent, tile, B, H, windows)
    o, lse = sta.sta_attention(q.cuda(), k.cuda(), v.cuda(), plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, scale)
    compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
            what=f"sharp x{factor}")


# ---------------------------------------------------------------- fused raster path

@pytest.mark.parametrize("latent,tile,B,H,d,windows", [
    ((18, 24, 24), (6, 8, 8), 1, 2, 64, [(12, 16, 16)] * 2),      # 2 (h, w) slices per block
    ((30, 48, 80), (6, 8, 8), 1, 2, 128, [(18, 24, 24), (30, 40, 40)]),
    ((8, 16, 24), (4, 8, 8), 2, 1, 128, [(8, 16, 16)]),            # 256-token tiles
    ((4, 16, 32), (1, 8, 16), 1, 2, 64, [(2, 8, 32), (4, 16, 16)]),  # one slice per block
    ((4, 32, 32), (2, 16, 16), 1, 1, 128, [(2, 32, 32)]),          # half a slice per block
])
def test_fused_raster_path_matches_permuted_path_bit_for_bit(sta, latent, tile, B, H, d, windows):
    assert sta.raster_supported(tile)
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator(device="cuda").manual_seed(N + d)
    q, k, v = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(3))
    plan = sta.sta_plan(latent, tile, B, H, windows)
    o1, l1 = sta.sta_attention(q, k, v, plan, 1.0 / math.sqrt(d), fused=True)
    o2, l2 = sta.sta_attention(q, k, v, plan, 1.0 / math.sqrt(d), fused=False)
    assert sta.sta_last_device_status(plan) == 0
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


def test_fused_raster_path_matches_oracle(sta):
    latent, tile, B, H, d = (4, 32, 32), (2, 16, 16), 1, 2, 64
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(77)
    q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
    windows = [(2, 16, 32), (4, 32, 16)]
    plan = sta.sta_plan(latent, tile, B, H, windows)
    o = torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda")
    lse = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    sta.sta_forward_raster(plan, q.cuda(), k.cuda(), v.cuda(), o, lse, 0.125)
    assert sta.sta_last_device_status(plan) == 0
    o_ref, lse_ref = oracle.sta_attention(q, k, v, latent, tile, windows, 0.125)
    compare(o.cpu().reshape(-1, d), lse.cpu().reshape(-1), o_ref.reshape(-1, d), lse_ref.reshape(-1),
            what="raster")


def test_fused_raster_rejects_unsupported_tiles(sta):
    tile = (8, 4, 12)  # 384 tokens, but a 128-row block is not a box of whole rows / slices
    assert not sta.raster_supported(tile)
    latent = (8, 8, 24)
    N = latent[0] * latent[1] * latent[2]
    plan = sta.sta_plan(latent, tile, 1, 1, [tile])
    x = torch.zeros(1, 1, N, 64, dtype=torch.bfloat16, device="cuda")
    lse = torch.zeros(1, 1, N, dtype=torch.float32, device="cuda")
    with pytest.raises(sta.StaError) as e:
        sta.sta_forward_raster(plan, x, x, x, torch.empty_like(x), lse, 0.125)
    assert e.value.status == sta.STA_ERR_UNSUPPORTED
    o, l = sta.sta_attention(x, x, x, plan, 0.125)   # runs the reorder / forward / unreorder kernels
    assert sta.sta_last_device_status(plan) == 0
    assert torch.count_nonzero(o).item() == 0


@pytest.mark.parametrize("latent", [(18, 24, 24), (13, 21, 18)])
def test_empty_batch_is_a_no_op(sta, latent):
    """B = 0: every call returns empty results without launching, for
    divisible and padded latents, through the plan, the fused and the permuted
    paths, the backward, autograd, the window statistics and the
    no-allocation forward; a later non-empty call on the device is unaffected."""
    tile, H, d = (6, 8, 8), 2, 64
    N = latent[0] * latent[1] * latent[2]
    plan = sta.sta_plan(latent, tile, 0, H, [(12, 16, 16)] * H)
    assert plan.flops(d) == 0
    q = torch.empty(0, H, N, d, device="cuda", dtype=torch.bfloat16)
    for fused in (True, False):
        o, lse = sta.sta_attention(q, q, q, plan, fused=fused)
        assert o.shape == q.shape and tuple(lse.shape) == (0, H, N)
        dq, dk, dv = sta.sta_attention_backward(q, q, q, o, lse, q, plan, fused=fused)
        assert dq.shape == dk.shape == dv.shape == q.shape
    qq = q.clone().requires_grad_(True)
    sta.StaAttention.apply(qq, qq, qq, plan).sum().backward()
    assert qq.grad.shape == q.shape
    r, m = sta.sta_window_stats(lse, lse, o, o)
    assert tuple(r.shape) == (0, H) and tuple(m.shape) == (0, H)
    if latent == (18, 24, 24):
        lse0 = torch.empty(0, H, N, device="cuda", dtype=torch.float32)
        sta.sta_forward_noalloc(latent, tile, 0, H, [(12, 16, 16)] * H, q, q, q, q.clone(), lse0, 0.125)
    assert sta.sta_last_device_status(plan) == 0
    plan.destroy()
    # the next real call runs normally
    w = sta_inputs.WORKLOADS[1]
    qa, ka, va = (x.cuda() for x in sta_inputs.make_qkv(w))
    p1 = sta.sta_plan(w.latent, w.tile, w.batch, w.heads, sta_inputs.windows(w).tolist())
    o1, l1 = sta.sta_attention(qa, ka, va, p1, w.softmax_scale)
    assert sta.sta_last_device_status(p1) == 0
    assert bool(torch.isfinite(o1.float()).all()) and bool(torch.isfinite(l1).all())
