"""The allocation-free forward, sta_forward_noalloc, against sta_forward and the oracle.

Callers whose device memory belongs to another allocator or pool, or that
reserve all their memory at start-up and may not allocate while serving, cannot
let sta_plan call cudaMalloc.  sta_forward_noalloc serves them by keeping its
plan in a fixed scratch array inside the library.  This test calls it through
the C ABI three times in a row on different problems (a small one, a larger one
with two batches and per-head windows of equal and different lengths, then the
small one again over what the larger one left in the scratch), and checks each
result against the plan-based sta_forward within the parity tolerance of the
other GPU tests, and sampled rows against the fp64 oracle.  It sits in a file
of its own that pytest collects last.
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import oracle
from parity_util import LSE_REL_TOL, O_MEAN_TOL, compare, o_bound, sample_tiles, tile_rows

pytestmark = pytest.mark.gpu

CASES = [
    ((18, 24, 24), (6, 8, 8), 1, 2, 64, [(12, 16, 16)] * 2),
    # windows of 27, 125 and again 27 tiles (another shape): the work list is
    # ordered by list length, ties by batch then head
    ((30, 48, 80), (6, 8, 8), 2, 4, 128, [(18, 24, 24), (30, 40, 40), (6, 24, 72), (18, 24, 24)]),
]


def check_close(o, lse, o_ref, lse_ref):
    do = (o.double() - o_ref.double()).abs()
    assert bool((do <= o_bound(o_ref.double())).all()), float(do.max())
    assert float(do.mean()) <= O_MEAN_TOL
    dl = (lse.double() - lse_ref.double()).abs() / lse_ref.double().abs().clamp_min(1.0)
    assert float(dl.max()) <= LSE_REL_TOL


def test_noalloc_forward_matches_plan_forward_and_oracle_on_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as sta
    lib = sta._lib
    stream = torch.cuda.current_stream()
    for call, i in enumerate([0, 1, 0]):
        latent, tile, B, H, d, windows = CASES[i]
        N = latent[0] * latent[1] * latent[2]
        g = torch.Generator().manual_seed(100 + i)
        q, k, v = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(3))
        scale = 1.0 / math.sqrt(d)
        # tile-major copies (the no-allocation forward takes tile-major tensors)
        qt, kt, vt = (torch.empty(B, H, N, d, dtype=torch.bfloat16, device="cuda") for _ in range(3))
        for x, y in zip((q, k, v), (qt, kt, vt)):
            sta.sta_tile_reorder(x.cuda(), y, latent, tile)
        # existing entry point: plan in device memory allocated by sta_plan
        plan = sta.sta_plan(latent, tile, B, H, windows)
        o_ref = torch.empty_like(qt)
        lse_ref = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        sta.sta_forward(plan, qt, kt, vt, o_ref, lse_ref, scale)
        assert sta.sta_last_device_status(plan) == 0
        # the allocation-free entry point, called through the C ABI
        o = torch.full_like(qt, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        geom = sta._geom(latent, tile)
        wins = (ctypes.c_int32 * (3 * H))(*[x for w in windows for x in w])
        st = lib.sta_forward_noalloc(ctypes.byref(geom), B, H, wins,
                                     ctypes.c_void_p(qt.data_ptr()), ctypes.c_void_p(kt.data_ptr()),
                                     ctypes.c_void_p(vt.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                     ctypes.c_void_p(lse.data_ptr()), d, scale,
                                     ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, sta.sta_status_string(st)
        torch.cuda.synchronize()
        check_close(o, lse, o_ref, lse_ref)
        # sampled rows against the oracle (raster order)
        o_r = torch.empty_like(o)
        lse_r = torch.empty_like(lse)
        sta.sta_tile_unreorder(o, o_r, latent, tile)
        sta.sta_tile_unreorder(lse, lse_r, latent, tile, token_dim=2)
        toks = tile_rows(latent, tile, sample_tiles(latent, tile, 1, seed=call), 8, seed=call)
        bhs = sorted({0, B * H - 1, H // 2})
        rows = np.array([(bh, t) for bh in bhs for t in toks], dtype=np.int64)
        o_want, lse_want = oracle.sta_attention(q, k, v, latent, tile, windows, scale, rows=rows)
        idx_bh, idx_t = torch.from_numpy(rows[:, 0]).cuda(), torch.from_numpy(rows[:, 1]).cuda()
        og = o_r.reshape(-1, N, d)[idx_bh, idx_t].cpu()
        lg = lse_r.reshape(-1, N)[idx_bh, idx_t].cpu()
        compare(og, lg, o_want, lse_want, what=f"no-allocation forward, call {call + 1}")
        plan.destroy()
