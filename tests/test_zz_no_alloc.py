"""The allocation-free forward, sta_forward_noalloc, against sta_forward.

Callers whose device memory belongs to another allocator or pool, or that
reserve all their memory at start-up and may not allocate while serving, cannot
let sta_plan call cudaMalloc.  sta_forward_noalloc serves them by keeping its
plan in a fixed scratch array inside the library.  This test calls it through
the C ABI twice in a row, on two different problems (so the second call runs
over what the first left in the scratch), and checks each result against the
plan-based sta_forward within the parity tolerance of the other GPU tests.
It sits in a file of its own that pytest collects last.
"""
import ctypes
import math

import pytest
import torch

from parity_util import LSE_REL_TOL, O_MEAN_TOL, o_bound

pytestmark = pytest.mark.gpu

CASES = [
    ((18, 24, 24), (6, 8, 8), 1, 2, 64, [(12, 16, 16)] * 2),
    ((30, 48, 80), (6, 8, 8), 1, 3, 128, [(18, 24, 24), (30, 40, 40), (30, 48, 80)]),
]


def check_close(o, lse, o_ref, lse_ref):
    do = (o.double() - o_ref.double()).abs()
    bound = o_bound(o_ref.double())
    assert bool((do <= bound).all()), float(do.max())
    assert float(do.mean()) <= O_MEAN_TOL
    dl = (lse.double() - lse_ref.double()).abs() / lse_ref.double().abs().clamp_min(1.0)
    assert float(dl.max()) <= LSE_REL_TOL


def test_noalloc_forward_matches_plan_forward_on_two_calls_in_a_row():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as sta
    lib = sta._lib
    stream = torch.cuda.current_stream()
    for i, (latent, tile, B, H, d, windows) in enumerate(CASES):
        N = latent[0] * latent[1] * latent[2]
        g = torch.Generator(device="cuda").manual_seed(100 + i)
        q, k, v = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16)
                   for _ in range(3))
        scale = 1.0 / math.sqrt(d)
        # existing entry point: plan in device memory allocated by sta_plan
        plan = sta.sta_plan(latent, tile, B, H, windows)
        o_ref = torch.empty_like(q)
        lse_ref = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
        sta.sta_forward(plan, q, k, v, o_ref, lse_ref, scale)
        assert sta.sta_last_device_status(plan) == 0
        # new entry point, called through the C ABI
        o = torch.full_like(q, float("nan"))
        lse = torch.full_like(lse_ref, float("nan"))
        geom = sta._geom(latent, tile)
        wins = (ctypes.c_int32 * (3 * H))(*[x for w in windows for x in w])
        st = lib.sta_forward_noalloc(ctypes.byref(geom), B, H, wins,
                                     ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                     ctypes.c_void_p(v.data_ptr()), ctypes.c_void_p(o.data_ptr()),
                                     ctypes.c_void_p(lse.data_ptr()), d, scale,
                                     ctypes.c_void_p(stream.cuda_stream))
        assert st == 0, sta.sta_status_string(st)
        torch.cuda.synchronize()
        check_close(o, lse, o_ref, lse_ref)
        plan.destroy()
