"""Host-side checks of the C-ABI library (no GPU, no compute call).

- the library loads and exports every function ``include/sta.h`` declares;
- argument validation happens before any launch;
- the plan's key-tile lists equal the sets derived from the oracle's
  token-level mask (bit-exact), for every workload geometry and window;
- the work list covers every (b, h, 128-row block) holding a real token
  exactly once (blocks of padding rows only are left out).
"""
import ctypes
import os
import re

import numpy as np
import pytest

import oracle
import sta_inputs
import sparse_attention_video_sta_b200 as sta

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_functions():
    src = open(os.path.join(ROOT, "include", "sta.h")).read()
    return sorted(set(re.findall(r"^STA_API\s+[\w\s\*]+?\b(sta_\w+)\s*\(", src, re.M)))


def test_library_exports_every_declared_symbol():
    names = declared_functions()
    assert len(names) >= 10
    lib = ctypes.CDLL(sta.library_path())
    for n in names:
        assert hasattr(lib, n), n
    assert set(names) == set(sta.EXPORTED_SYMBOLS)


def test_status_strings():
    assert sta.sta_status_string(0) == "STA_OK"
    assert sta.sta_status_string(4) == "STA_ERR_TIMEOUT"
    assert sta.sta_status_string(99) == "STA_ERR_UNKNOWN"


def _raw_plan_host(latent, tile, batch, heads, windows):
    lib = sta._lib
    g = sta._geom(latent, tile)
    h = ctypes.c_void_p(0)
    w = (ctypes.c_int32 * (3 * heads))(*[int(x) for win in windows for x in win])
    st = lib.sta_plan_host(ctypes.byref(g), batch, heads, w, ctypes.byref(h))
    return st, h


def test_plan_argument_validation():
    INV, UNS = sta.STA_ERR_INVALID_ARG, sta.STA_ERR_UNSUPPORTED
    assert _raw_plan_host((30, 48, 80), (6, 8, 8), 1, 1, [(18, 24, 24)])[0] == 0
    # a latent axis that is not a multiple of the tile is padded to whole tiles
    assert _raw_plan_host((30, 48, 81), (6, 8, 8), 1, 1, [(18, 24, 24)])[0] == 0
    assert _raw_plan_host((33, 45, 80), (6, 8, 8), 1, 1, [(18, 24, 24)])[0] == 0
    assert _raw_plan_host((30, 48, 0), (6, 8, 8), 1, 1, [(18, 24, 24)])[0] == INV
    assert _raw_plan_host((30, 48, 80), (6, 0, 8), 1, 1, [(18, 24, 24)])[0] == INV
    assert _raw_plan_host((30, 48, 80), (6, 8, 8), 1, 1, [(18, 24, 20)])[0] == INV  # window % tile
    assert _raw_plan_host((30, 48, 80), (6, 8, 8), 1, 1, [(0, 24, 24)])[0] == INV
    assert _raw_plan_host((30, 48, 80), (6, 8, 8), -1, 1, [(18, 24, 24)])[0] == INV
    assert _raw_plan_host((30, 48, 80), (6, 8, 8), 1, 0, [])[0] == INV
    assert _raw_plan_host((30, 48, 80), (3, 8, 8), 1, 1, [(18, 24, 24)])[0] == UNS  # 192 tokens
    # int32 row-coordinate limit of the kernel's tensor maps
    assert _raw_plan_host((96, 512, 512), (6, 8, 8), 2, 48, [(18, 24, 24)] * 48)[0] == UNS
    lib = sta._lib
    assert lib.sta_plan_host(None, 1, 1, None, None) == INV
    assert lib.sta_plan_destroy(None) == 0


def test_calls_rejected_before_launch():
    INV = sta.STA_ERR_INVALID_ARG
    lib = sta._lib
    g = sta._geom((18, 24, 24), (6, 8, 8))
    bad = sta._geom((18, 24, 0), (6, 8, 8))
    p = ctypes.c_void_p(1 << 20)
    assert lib.sta_tile_reorder(None, p, 1, 128, ctypes.byref(g), None) == INV
    assert lib.sta_tile_reorder(p, None, 1, 128, ctypes.byref(g), None) == INV
    assert lib.sta_tile_reorder(p, ctypes.c_void_p((1 << 20) + 64), 1, 128, ctypes.byref(g), None) == INV
    assert lib.sta_tile_reorder(p, ctypes.c_void_p(1 << 34), -1, 128, ctypes.byref(g), None) == INV
    assert lib.sta_tile_reorder(p, ctypes.c_void_p(1 << 34), 1, 0, ctypes.byref(g), None) == INV
    assert lib.sta_tile_unreorder(p, ctypes.c_void_p(1 << 34), 1, 128, ctypes.byref(bad), None) == INV
    # forward: host-only plan, null / misaligned pointers, bad scale, bad head_dim
    hp = sta.sta_plan_host((18, 24, 24), (6, 8, 8), 1, 2, [(12, 16, 16)] * 2)
    a = ctypes.c_void_p(1 << 30)
    assert lib.sta_forward(hp.handle, a, a, a, a, a, 64, 0.125, None) == INV
    assert lib.sta_forward(None, a, a, a, a, a, 64, 0.125, None) == INV
    assert lib.sta_last_device_status(hp.handle, None) == INV
    assert lib.sta_debug_inject_timeout(1, 0) == INV
    assert lib.sta_debug_inject_timeout(3, 30) == INV
    assert lib.sta_debug_inject_timeout(-1, 30) == INV
    assert lib.sta_plan_query(hp.handle, 2, 0, None, 0, ctypes.byref(ctypes.c_int32())) == INV
    assert lib.sta_plan_query(hp.handle, 0, 27, None, 0, ctypes.byref(ctypes.c_int32())) == INV
    hp.destroy()


def oracle_tile_set(latent, tile, window, q_tile):
    """Key tiles attended by query tile q_tile, read off the oracle's token mask."""
    toks = oracle.tile_tokens(latent, tile, q_tile)
    row = oracle.mask_row(latent, tile, window, int(toks[0]))
    n_tiles = oracle.num_tokens(latent) // (tile[0] * tile[1] * tile[2])
    out = []
    for t in range(n_tiles):
        kt = oracle.tile_tokens(latent, tile, t)
        blk = row[kt]
        assert blk.all() or not blk.any()
        if blk.all():
            out.append(t)
    return out


@pytest.mark.parametrize("idx", [1, 2, 3, 4, 5])
def test_plan_lists_match_oracle_mask(idx):
    w = sta_inputs.WORKLOADS[idx]
    wins = sta_inputs.windows(w).tolist()
    p = sta.sta_plan_host(w.latent, w.tile, w.batch, w.heads, wins)
    n_tiles = p.tiles_per_head
    rng = np.random.default_rng(idx)
    distinct = {}
    for h, win in enumerate(wins):
        distinct.setdefault(tuple(win), h)
    for win, h in distinct.items():
        tiles = sorted(set([0, n_tiles - 1, n_tiles // 2] + rng.integers(0, n_tiles, 6).tolist()))
        if n_tiles <= 30:
            tiles = range(n_tiles)
        for q in tiles:
            assert p.query(h, q) == oracle_tile_set(w.latent, w.tile, win, q), (idx, win, q)
    pairs, items = p.stats()
    expect = 0
    vol = w.tile[0] * w.tile[1] * w.tile[2]
    for win in wins:
        e = [min(win[i] // w.tile[i], w.latent[i] // w.tile[i]) for i in range(3)]
        expect += n_tiles * e[0] * e[1] * e[2]
    assert pairs == expect * w.batch
    # the pages' 91% sparsity for w=(18,24,24) on the 720p latent
    if idx == 2:
        assert pairs == 300 * 27 * 24
        assert abs(1 - pairs / (24 * 300 * 300) - 0.91) < 1e-12
    assert items >= w.batch * w.heads * n_tiles * (vol // 128) // 2


def real_blocks(latent, tile):
    """Tile-major 128-row blocks holding at least one real token, read off the
    oracle's tile-major positions of the latent's tokens."""
    N = latent[0] * latent[1] * latent[2]
    return sorted(set((oracle.tile_major_index(latent, tile, np.arange(N)) // 128).tolist()))


def test_work_list_covers_every_row_block_once():
    for latent, tile, heads, batch in [((18, 24, 24), (6, 8, 8), 2, 1), ((12, 16, 16), (4, 8, 8), 3, 2),
                                       ((6, 16, 16), (2, 8, 8), 1, 1), ((30, 48, 80), (6, 8, 8), 24, 1),
                                       ((18, 24, 16), (6, 8, 8), 2, 2), ((33, 45, 80), (6, 8, 8), 3, 1),
                                       ((13, 21, 18), (6, 8, 8), 2, 2), ((1, 1, 1), (6, 8, 8), 1, 2)]:
        wins = [tuple(3 * t for t in tile)] * (heads - 1) + [tile]
        p = sta.sta_plan_host(latent, tile, batch, heads, wins)
        items = p.work_items()
        S = (tile[0] * tile[1] * tile[2]) // 128
        n_tiles = p.tiles_per_head
        seen = {}
        lens = []
        for bh, qa, qb, win in items:
            h = bh % heads
            assert qb == -1  # one query block per item
            assert 0 <= qa < n_tiles * S
            seen[(bh, qa)] = seen.get((bh, qa), 0) + 1
            lens.append(len(p.query(h, qa // S)))
        real = real_blocks(latent, tile)
        assert sorted(seen) == [(bh, r) for bh in range(batch * heads) for r in real]
        assert all(c == 1 for c in seen.values())
        assert lens == sorted(lens, reverse=True)  # longest lists first
        pairs, n_items = p.stats()
        assert n_items == len(items)


@pytest.mark.parametrize("idx", [1, 2, 3])
def test_key_lists_are_transposed_query_lists(idx):
    """sta_plan_key_query(kt) lists exactly the query tiles whose oracle mask
    attends tile kt (the backward's dK / dV kernel walks these lists)."""
    w = sta_inputs.WORKLOADS[idx]
    wins = sta_inputs.windows(w).tolist()
    p = sta.sta_plan_host(w.latent, w.tile, w.batch, w.heads, wins)
    n_tiles = p.tiles_per_head
    distinct = {}
    for h, win in enumerate(wins):
        distinct.setdefault(tuple(win), h)
    for win, h in distinct.items():
        attends = [set(oracle_tile_set(w.latent, w.tile, win, q)) for q in range(n_tiles)]
        for kt in range(n_tiles):
            expect = [q for q in range(n_tiles) if kt in attends[q]]
            assert p.key_query(h, kt) == expect, (idx, win, kt)


def test_backward_rejected_before_launch():
    INV = sta.STA_ERR_INVALID_ARG
    lib = sta._lib
    hp = sta.sta_plan_host((18, 24, 24), (6, 8, 8), 1, 2, [(12, 16, 16)] * 2)
    a = ctypes.c_void_p(1 << 30)
    args = [a] * 10
    assert lib.sta_backward(hp.handle, *args, 64, 0.125, None) == INV  # host-only plan
    assert lib.sta_backward(None, *args, 64, 0.125, None) == INV
    assert lib.sta_plan_key_query(hp.handle, 0, 27, None, 0, ctypes.byref(ctypes.c_int32())) == INV
    assert lib.sta_plan_key_query(hp.handle, 2, 0, None, 0, ctypes.byref(ctypes.c_int32())) == INV
    hp.destroy()


def test_window_stats_rejected_before_launch():
    INV = sta.STA_ERR_INVALID_ARG
    lib = sta._lib
    a = ctypes.c_void_p(1 << 30)
    odd = ctypes.c_void_p((1 << 30) + 8)
    assert lib.sta_window_stats(None, a, a, a, 1, 128, 64, a, a, None) == INV
    assert lib.sta_window_stats(a, a, odd, a, 1, 128, 64, a, a, None) == INV   # o not 16-byte aligned
    assert lib.sta_window_stats(a, a, a, a, -1, 128, 64, a, a, None) == INV    # negative slice count
    assert lib.sta_window_stats(a, a, a, a, 0, 128, 64, a, a, None) == 0       # no slices: a no-op
    assert lib.sta_window_stats(a, a, a, a, 1, 0, 64, a, a, None) == INV       # no tokens
    assert lib.sta_window_stats(a, a, a, a, 1, 128, 12, a, a, None) == INV     # head_dim not a multiple of 8


@pytest.mark.parametrize("latent,tile,windows", [
    ((13, 21, 18), (6, 8, 8), [(6, 8, 8), (12, 16, 16), (18, 24, 24)]),
    ((9, 8, 20), (4, 8, 8), [(8, 8, 16), (4, 8, 24)]),
])
def test_padded_plan_lists_match_oracle_mask(latent, tile, windows):
    """Latents that are not a multiple of the tile: the plan's lists (and the
    transposed lists) equal the tile sets read off the oracle's token mask."""
    p = sta.sta_plan_host(latent, tile, 1, len(windows), windows)
    n = [-(-latent[i] // tile[i]) for i in range(3)]
    n_tiles = n[0] * n[1] * n[2]
    assert p.tiles_per_head == n_tiles
    assert p.padded_tokens == n_tiles * tile[0] * tile[1] * tile[2]
    for h, win in enumerate(windows):
        attends = []
        for q in range(n_tiles):
            toks = oracle.tile_tokens(latent, tile, q)
            row = oracle.mask_row(latent, tile, win, int(toks[0]))
            got = []
            for t in range(n_tiles):
                blk = row[oracle.tile_tokens(latent, tile, t)]
                assert blk.all() or not blk.any()
                if blk.all():
                    got.append(t)
            assert p.query(h, q) == got, (latent, win, q)
            attends.append(set(got))
        for kt in range(n_tiles):
            assert p.key_query(h, kt) == [q for q in range(n_tiles) if kt in attends[q]]


def test_pipe_rejected_before_allocation():
    INV = sta.STA_ERR_INVALID_ARG
    lib = sta._lib
    hp = sta.sta_plan_host((18, 24, 24), (6, 8, 8), 1, 2, [(12, 16, 16)] * 2)
    out = ctypes.c_void_p(0)
    assert lib.sta_pipe_create(hp.handle, 64, 0.125, 2, ctypes.byref(out)) == INV  # host-only plan
    assert lib.sta_pipe_create(None, 64, 0.125, 2, ctypes.byref(out)) == INV
    assert lib.sta_pipe_create(hp.handle, 64, 0.125, 2, None) == INV
    assert lib.sta_pipe_submit(None, None, None, None, None, None) == INV
    assert lib.sta_pipe_wait(None) == INV
    assert lib.sta_pipe_destroy(None) == 0
    hp.destroy()


@pytest.mark.parametrize("latent,tile,heads,batch,wins", [
    ((30, 48, 80), (6, 8, 8), 24, 1, None),
    ((18, 24, 24), (6, 8, 8), 3, 2, [(6, 8, 8), (12, 16, 16), (18, 24, 24)]),
    ((13, 21, 18), (6, 8, 8), 2, 1, [(6, 8, 8), (18, 24, 24)]),
    ((33, 45, 80), (6, 8, 8), 24, 1, None),
])
def test_backward_work_lists(latent, tile, heads, batch, wins):
    """Each backward list holds every (b, h, block) with a real token once
    (blocks of padding rows only are left out); rounds of 148 items
    (one per CTA of the host plan's grid) keep natural (b, h, block) order
    between rounds, and per-CTA totals of list lengths stay level."""
    wins = wins or [(18, 24, 24)] * heads
    p = sta.sta_plan_host(latent, tile, batch, heads, wins)
    S = (tile[0] * tile[1] * tile[2]) // 128
    real = real_blocks(latent, tile)
    for which in (0, 1):
        items = p.backward_items(which)
        assert all(qb == -1 for _, _, qb, _ in items)
        keys = sorted((bh, blk) for bh, blk, _, _ in items)
        natural = [(bh, blk) for bh in range(batch * heads) for blk in real]
        assert keys == natural
        R = 148
        for r0 in range(0, len(items), R):
            assert sorted((bh, blk) for bh, blk, _, _ in items[r0:r0 + R]) == natural[r0:r0 + R]
        def length(it):
            bh, blk, _, win = it
            h = bh % heads
            t = blk // S
            return len(p.query(h, t)) if which == 0 else len(p.key_query(h, t))
        # after every full round the CTAs' totals differ by at most one item
        # (a final partial round can only go to the first CTAs of the grid)
        loads = [0] * R
        longest = max(length(it) for it in items)
        for r0 in range(0, len(items) - R + 1, R):
            for c, it in enumerate(items[r0:r0 + R]):
                loads[c] += length(it)
            assert max(loads) - min(loads) <= longest, (which, r0, max(loads), min(loads))


def test_empty_problems_are_no_ops():
    """Batch 0 (and outer 0, slices 0): the other arguments are still checked,
    nothing is launched, STA_OK is returned and the tensor pointers (null for
    an empty PyTorch tensor) are not read."""
    INV, UNS = sta.STA_ERR_INVALID_ARG, sta.STA_ERR_UNSUPPORTED
    lib = sta._lib
    st, h = _raw_plan_host((18, 24, 24), (6, 8, 8), 0, 2, [(12, 16, 16), (18, 24, 24)])
    assert st == 0
    pairs, items = ctypes.c_int64(-1), ctypes.c_int64(-1)
    assert lib.sta_plan_stats(h, ctypes.byref(pairs), ctypes.byref(items)) == 0
    assert pairs.value == 0 and items.value == 0
    for which in (0, 1):
        cnt = ctypes.c_int64(-1)
        assert lib.sta_plan_backward_items(h, which, None, 0, ctypes.byref(cnt)) == 0
        assert cnt.value == 0
    # the key-tile lists still exist: they do not depend on the batch
    ids = (ctypes.c_int32 * 27)()
    cnt32 = ctypes.c_int32(-1)
    assert lib.sta_plan_query(h, 1, 13, ids, 27, ctypes.byref(cnt32)) == 0 and cnt32.value == 27
    assert lib.sta_plan_destroy(h) == 0
    g = sta._geom((18, 24, 24), (6, 8, 8))
    bad = sta._geom((18, 24, 0), (6, 8, 8))
    assert lib.sta_tile_reorder(None, None, 0, 256, ctypes.byref(g), None) == 0
    assert lib.sta_tile_unreorder(None, None, 0, 256, ctypes.byref(g), None) == 0
    assert lib.sta_tile_reorder(None, None, 0, 256, ctypes.byref(bad), None) == INV
    assert lib.sta_tile_reorder(None, None, 0, 0, ctypes.byref(g), None) == INV
    f64 = ctypes.POINTER(ctypes.c_double)
    assert lib.sta_window_stats(None, None, None, None, 0, 100, 128, None, None, None) == 0
    assert lib.sta_window_stats(None, None, None, None, 0, 0, 128, None, None, None) == INV
    assert lib.sta_window_stats(None, None, None, None, -1, 100, 128, None, None, None) == INV
    assert lib.sta_window_stats(None, None, None, None, 1, 100, 128, None, None, None) == INV
    # the no-allocation forward: batch 0 is a no-op; a padded latent is unsupported
    w = (ctypes.c_int32 * 3)(12, 16, 16)
    assert lib.sta_forward_noalloc(ctypes.byref(g), 0, 1, w, None, None, None, None, None, 128,
                                   ctypes.c_float(0.088), None) == 0
    assert lib.sta_forward_noalloc(ctypes.byref(g), 0, 1, w, None, None, None, None, None, 96,
                                   ctypes.c_float(0.088), None) == UNS
    assert lib.sta_forward_noalloc(ctypes.byref(g), 0, 1, w, None, None, None, None, None, 128,
                                   ctypes.c_float(0.0), None) == INV
    pad = sta._geom((18, 24, 20), (6, 8, 8))
    assert lib.sta_forward_noalloc(ctypes.byref(pad), 1, 1, w, None, None, None, None, None, 128,
                                   ctypes.c_float(0.088), None) == UNS
    assert lib.sta_forward_noalloc(ctypes.byref(g), -1, 1, w, None, None, None, None, None, 128,
                                   ctypes.c_float(0.088), None) == INV
    assert lib.sta_forward_noalloc(ctypes.byref(g), 1, 1, w, None, None, None, None, None, 128,
                                   ctypes.c_float(0.088), None) == INV


def test_noalloc_limits_rejected_before_any_cuda_call():
    """The allocation-free forward rejects problems beyond its fixed scratch
    (more than 1024 heads, or a plan image above 4 MiB) with UNSUPPORTED
    before it looks up the scratch or launches anything, so the placeholder
    (never dereferenced) tensor addresses below are safe on any machine."""
    lib = sta._lib
    UNS = 2
    g = sta._geom((30, 48, 80), (6, 8, 8))
    fake = ctypes.c_void_p(1 << 20)
    lse = ctypes.cast(fake, ctypes.POINTER(ctypes.c_float))
    scale = ctypes.c_float(0.088)
    heads = 1025
    w = (ctypes.c_int32 * (3 * heads))(*([18, 24, 24] * heads))
    assert lib.sta_forward_noalloc(ctypes.byref(g), 1, heads, w, fake, fake, fake, fake, lse, 128,
                                   scale, None) == UNS
    # 1024 heads of the 720p latent: 460 800 two-block items, 7.4 MB of plan
    heads = 1024
    w = (ctypes.c_int32 * (3 * heads))(*([18, 24, 24] * heads))
    assert lib.sta_forward_noalloc(ctypes.byref(g), 1, heads, w, fake, fake, fake, fake, lse, 128,
                                   scale, None) == UNS


def test_device_helper_requires_one_cuda_device():
    """The binding's device check (no GPU needed): host tensors alone name no
    CUDA device; a plan's device is used when no tensor is given."""
    import torch
    with pytest.raises(ValueError, match="one CUDA device"):
        sta._device((torch.zeros(1),))
    p = sta.sta_plan_host((18, 24, 24), (6, 8, 8), 1, 1, [(12, 16, 16)])
    assert p.device is None
    p.device = 3
    assert sta._device((), p) == torch.device("cuda", 3)
    p.device = None
    p.destroy()
