"""The debug build (libsta_debug.so): device-side checks of every plan index.

Its kernels check each work item and the key-tile list it names before any
load or product uses them (csrc/sta_bounds.cuh).  On a clean plan the debug
build must give the same bits as the regular one and leave the status word
clear; with one key-tile id of the device plan moved past the tile grid (the
debug hook sta_debug_plan_poke) the forward and the backward's dQ kernel must
stop and report STA_ERR_BOUNDS, and the next call on the restored plan must be
clean again.  The corrupted id is only ever used, unchecked, as the row of a
tile-major TMA box, which the TMA unit fills with zeros outside the tensor:
even a check that failed to fire could not make an out-of-bounds access.
"""
import ctypes
import math
import os

import pytest
import torch

import sparse_attention_video_sta_b200 as sta

pytestmark = pytest.mark.gpu


def debug_lib():
    path = os.path.join(os.path.dirname(sta.library_path()), "libsta_debug.so")
    if not os.path.exists(path):
        import importlib.util
        spec = importlib.util.spec_from_file_location(
            "_sta_build", os.path.join(os.path.dirname(sta.library_path()), "_build.py"))
        mod = importlib.util.module_from_spec(spec)
        spec.loader.exec_module(mod)
        mod.build(debug=True)
    L = ctypes.CDLL(path)
    vp, i32, i64 = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64
    G = ctypes.POINTER(sta._Geom)
    i32p = ctypes.POINTER(ctypes.c_int32)
    sig = {
        "sta_plan": [G, i32, i32, i32p, vp, ctypes.POINTER(vp)],
        "sta_plan_destroy": [vp],
        "sta_plan_query": [vp, i32, i32, i32p, i32, i32p],
        "sta_forward": [vp, vp, vp, vp, vp, vp, i32, ctypes.c_float, vp],
        "sta_backward": [vp] * 11 + [i32, ctypes.c_float, vp],
        "sta_last_device_status": [vp, vp],
        "sta_debug_plan_poke": [vp, i32, i64, i32],
    }
    for name, args in sig.items():
        f = getattr(L, name)
        f.argtypes = args
        f.restype = ctypes.c_int
    return L


def test_debug_build_is_clean_and_reports_a_corrupted_plan_index():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    L = debug_lib()
    latent, tile, B, H, d = (30, 48, 80), (6, 8, 8), 1, 2, 128
    windows = [(18, 24, 24), (30, 40, 40)]
    N = latent[0] * latent[1] * latent[2]
    scale = 1.0 / math.sqrt(d)
    g = torch.Generator(device="cuda").manual_seed(31)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(4))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    ptr = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    # regular build, through the package (tile-major tensors)
    ref_plan = sta.sta_plan(latent, tile, B, H, windows)
    o_ref = torch.empty_like(q)
    l_ref = torch.empty(B, H, N, dtype=torch.float32, device="cuda")
    sta.sta_forward(ref_plan, q, k, v, o_ref, l_ref, scale)
    assert sta.sta_last_device_status(ref_plan) == 0
    # debug build through its own C ABI
    geom = sta._geom(latent, tile)
    wins = (ctypes.c_int32 * (3 * H))(*[x for w in windows for x in w])
    plan = ctypes.c_void_p()
    assert L.sta_plan(ctypes.byref(geom), B, H, wins, stream, ctypes.byref(plan)) == 0
    o, lse = torch.empty_like(q), torch.empty_like(l_ref)

    def forward():
        assert L.sta_forward(plan, ptr(q), ptr(k), ptr(v), ptr(o), ptr(lse), d, scale, stream) == 0
        return L.sta_last_device_status(plan, stream)

    assert forward() == sta.STA_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    # entry 5 of query tile 0's key list (head 0) moved one past the grid
    lst = (ctypes.c_int32 * 64)()
    cnt = ctypes.c_int32(0)
    assert L.sta_plan_query(plan, 0, 0, lst, 64, ctypes.byref(cnt)) == 0 and cnt.value == 27
    tiles = (latent[0] // tile[0]) * (latent[1] // tile[1]) * (latent[2] // tile[2])
    assert L.sta_debug_plan_poke(plan, 0, 5, tiles) == 0
    assert forward() == sta.STA_ERR_BOUNDS
    dq, dk, dv = (torch.empty_like(q) for _ in range(3))
    ws = torch.empty(2 * B * H * N, dtype=torch.float32, device="cuda")
    assert L.sta_backward(plan, ptr(q), ptr(k), ptr(v), ptr(o_ref), ptr(do), ptr(l_ref), ptr(dq), ptr(dk),
                          ptr(dv), ptr(ws), d, scale, stream) == 0
    assert L.sta_last_device_status(plan, stream) == sta.STA_ERR_BOUNDS
    # restored: clean again, same bits as the regular build
    assert L.sta_debug_plan_poke(plan, 0, 5, lst[5]) == 0
    assert forward() == sta.STA_OK
    assert torch.equal(o, o_ref) and torch.equal(lse, l_ref)
    assert L.sta_plan_destroy(plan) == 0
    ref_plan.destroy()
