"""Host-side plan validation (sta_plan_validate) and the debug library.

Every plan is checked when it is built: CSR offsets non-decreasing and inside
the id arrays, tile ids inside the grid, work items inside their (b, h), row
block and window ranges, the transposed lists the exact transpose of the
forward lists, tile origins inside the padded latent.  These tests build plans
on the host, check that they validate, then corrupt one entry at a time
through the debug hook and check that validation names the violation.  They
also check that the debug build (kernels with device-side index checks) loads
and exports the same C ABI.  CPU only.
"""
import ctypes
import os

import pytest

import sparse_attention_video_sta_b200 as sta

INV = sta.STA_ERR_INVALID_ARG


def host_plan(latent, tile, B, H, windows):
    return sta.sta_plan_host(latent, tile, B, H, windows)


@pytest.mark.parametrize("latent,tile,B,H,windows", [
    ((30, 48, 80), (6, 8, 8), 1, 3, [(18, 24, 24), (30, 40, 40), (30, 48, 80)]),
    ((13, 21, 18), (6, 8, 8), 2, 2, [(6, 8, 8), (12, 16, 16)]),     # padded latent
    ((12, 16, 16), (4, 8, 8), 1, 2, [(4, 8, 8), (12, 16, 16)]),
])
def test_built_plans_validate(latent, tile, B, H, windows):
    p = host_plan(latent, tile, B, H, windows)
    p.validate()
    assert sta._lib.sta_plan_validate(p.handle) == sta.STA_OK
    p.destroy()


def poke(p, which, index, value):
    return sta._lib.sta_debug_plan_poke(p.handle, which, index, value)


def detail():
    return sta._lib.sta_last_error_detail().decode()


def test_corrupted_entries_are_caught():
    latent, tile = (30, 48, 80), (6, 8, 8)
    p = host_plan(latent, tile, 1, 2, [(18, 24, 24), (30, 40, 40)])
    tiles = p.tiles_per_head
    # a key-tile id past the grid
    old = p.query(0, 0)[0]
    assert poke(p, 0, 0, tiles) == sta.STA_OK
    assert sta._lib.sta_plan_validate(p.handle) == INV and "csr_ids" in detail()
    assert poke(p, 0, 0, old) == sta.STA_OK
    p.validate()
    # a key-tile id inside the grid but not in the transposed lists
    assert poke(p, 0, 0, tiles - 1) == sta.STA_OK
    assert sta._lib.sta_plan_validate(p.handle) == INV and "tcsr" in detail()
    assert poke(p, 0, 0, old) == sta.STA_OK
    # a work item of a (b, h) that does not exist, and a window id out of range
    items = p.work_items()
    assert poke(p, 1, 0, 2) == sta.STA_OK
    assert sta._lib.sta_plan_validate(p.handle) == INV and "f1_items" in detail()
    assert poke(p, 1, 0, int(items[0][0])) == sta.STA_OK
    assert poke(p, 1, 3, 7) == sta.STA_OK
    assert sta._lib.sta_plan_validate(p.handle) == INV
    assert poke(p, 1, 3, int(items[0][3])) == sta.STA_OK
    p.validate()
    # offsets out of order
    assert poke(p, 2, 1, -1) == sta.STA_OK
    assert sta._lib.sta_plan_validate(p.handle) == INV and "csr_off" in detail()
    p.destroy()


def test_poke_rejects_bad_arguments():
    p = host_plan((18, 24, 24), (6, 8, 8), 1, 1, [(12, 16, 16)])
    assert poke(p, 4, 0, 0) == INV
    assert poke(p, 0, -1, 0) == INV
    assert poke(p, 0, 10 ** 9, 0) == INV
    assert sta._lib.sta_plan_validate(None) == INV
    p.destroy()


def test_debug_library_exports_the_same_abi():
    path = os.path.join(os.path.dirname(sta.library_path()), "libsta_debug.so")
    assert os.path.exists(path), "libsta_debug.so missing: run __graft_entry__.build()"
    lib = ctypes.CDLL(path)
    for name in sta.EXPORTED_SYMBOLS:
        assert hasattr(lib, name), name
