"""GPU parity of the STA backward pass (dQ, dK, dV) against the fp64 oracle.

The CUDA path runs as a user would: the fused forward on raster tensors gives
O and LSE, then the backward (through ``sta_attention_backward``: permutation
to tile-major order, ``sta_backward`` through the C ABI, permutation back).
Expected values come only from ``oracle``; tolerances are in ``parity_util``.
"""
import numpy as np
import pytest
import torch

import oracle
import sta_inputs
from parity_util import compare_grad, sample_tiles, tile_rows

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as s
    return s


def gpu_grads(sta, q, k, v, do, latent, tile, windows, scale):
    B, H = q.shape[0], q.shape[1]
    plan = sta.sta_plan(latent, tile, B, H, windows)
    qd, kd, vd, dod = q.cuda(), k.cuda(), v.cuda(), do.cuda()
    o, lse = sta.sta_attention(qd, kd, vd, plan, scale)
    dq, dk, dv = sta.sta_attention_backward(qd, kd, vd, o, lse, dod, plan, scale)
    assert sta.sta_last_device_status(plan) == 0
    return plan, dq, dk, dv


def rows_of(t, rows):
    flat = t.reshape(-1, t.shape[2], t.shape[3])
    return flat[torch.from_numpy(rows[:, 0]).to(t.device), torch.from_numpy(rows[:, 1]).to(t.device)].cpu()


def check_all_rows(sta, latent, tile, B, H, d, windows, scale, seed):
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(seed)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4))
    _, dq, dk, dv = gpu_grads(sta, q, k, v, do, latent, tile, windows, scale)
    rq, rk, rv = oracle.sta_backward(q, k, v, do, latent, tile, windows, scale)
    bh = np.repeat(np.arange(B * H), N)
    out = {}
    for name, a, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        out[name] = compare_grad(a.cpu().reshape(-1, d), r.reshape(-1, d), bh, what=f"{name} {latent} {windows}")
    return out


def test_backward_tiny_workload_all_rows(sta):
    w = sta_inputs.WORKLOADS[1]
    q, k, v = sta_inputs.make_qkv(w)
    do = sta_inputs.make_dout(w)
    wins = sta_inputs.windows(w).tolist()
    _, dq, dk, dv = gpu_grads(sta, q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    rq, rk, rv = oracle.sta_backward(q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    bh = np.repeat(np.arange(w.batch * w.heads), w.tokens)
    d = w.head_dim
    for name, a, r in (("dq", dq, rq), ("dk", dk, rk), ("dv", dv, rv)):
        compare_grad(a.cpu().reshape(-1, d), r.reshape(-1, d), bh, what=name)


@pytest.mark.parametrize("latent,tile,B,H,d,windows", [
    ((12, 16, 16), (6, 8, 8), 1, 2, 128, [[6, 8, 8], [12, 16, 16]]),          # one-tile window, full
    ((12, 16, 24), (6, 8, 8), 2, 3, 128, [[6, 16, 8], [12, 8, 24], [6, 8, 16]]),  # even extents
    ((18, 16, 32), (6, 8, 8), 1, 2, 64, [[18, 8, 16], [6, 16, 24]]),
    ((8, 16, 16), (2, 8, 8), 1, 2, 128, [[4, 8, 8], [8, 16, 8]]),            # one block per tile
    ((12, 16, 16), (4, 8, 8), 1, 1, 128, [[8, 8, 16]]),                      # two blocks per tile
])
def test_backward_small_geometries_all_rows(sta, latent, tile, B, H, d, windows):
    check_all_rows(sta, latent, tile, B, H, d, windows, 1.0 / np.sqrt(d), seed=sum(latent) + H + d)


def test_backward_long_transposed_lists_all_keys(sta):
    """Full window over a 5 x 4 x 5 grid of 6 x 8 x 8 tiles (100 tiles, 38 400
    tokens): every key block's transposed list holds all 100 query tiles, so
    the dK / dV kernel accumulates over 300 query blocks per item, the longest
    lists any element-wise check here reaches.  dK and dV at every key row,
    against the oracle (about a minute of host work on 16 cores)."""
    latent, tile, B, H, d = (30, 32, 40), (6, 8, 8), 1, 1, 128
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(4242)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16) for _ in range(4))
    windows = [list(latent)]
    scale = 1.0 / np.sqrt(d)
    plan, dq, dk, dv = gpu_grads(sta, q, k, v, do, latent, tile, windows, scale)
    assert len(plan.key_query(0, 0)) == 100 and len(plan.key_query(0, 57)) == 100
    rk, rv = oracle.sta_backward_dkdv(q, k, v, do, latent, tile, windows, scale)
    bh = np.repeat(np.arange(B * H), N)
    compare_grad(dk.cpu().reshape(-1, d), rk.reshape(-1, d), bh, what="dk full window, 100-tile lists")
    compare_grad(dv.cpu().reshape(-1, d), rv.reshape(-1, d), bh, what="dv full window, 100-tile lists")


def test_backward_720p_sampled(sta):
    """The 720p workload with window (18,24,24): dQ on sampled query rows of
    every tile class, dK / dV on sampled keys of corner, edge and centre tiles."""
    w = sta_inputs.WORKLOADS[2]
    heads = [0, 13]
    q, k, v = sta_inputs.make_qkv(w, device="cuda")
    do = sta_inputs.make_dout(w, device="cuda")
    wins = sta_inputs.windows(w).tolist()
    plan, dq, dk, dv = gpu_grads(sta, q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    qc, kc, vc, doc = (x.cpu() for x in (q, k, v, do))
    tiles = sample_tiles(w.latent, w.tile, 3, seed=5)
    toks = tile_rows(w.latent, w.tile, tiles, 6, seed=6)
    rows = np.array([(h, t) for h in heads for t in toks], dtype=np.int64)
    ref = oracle.sta_backward_dq(qc, kc, vc, doc, w.latent, w.tile, wins, w.softmax_scale, rows=rows)
    compare_grad(rows_of(dq, rows), ref, rows[:, 0], what="dq 720p")
    # keys: 12 tokens of each of three key tiles (corner, edge, interior), one head each
    n = [w.latent[i] // w.tile[i] for i in range(3)]
    key_tiles = [0, (n[0] // 2 * n[1] + 0) * n[2] + n[2] - 1, ((n[0] // 2) * n[1] + n[1] // 2) * n[2] + 4]
    rng = np.random.default_rng(7)
    keys = []
    for i, kt in enumerate(key_tiles):
        tt = oracle.tile_tokens(w.latent, w.tile, kt)
        for t in np.concatenate([tt[[0, 127, 128, 383]], rng.choice(tt, 8, replace=False)]):
            keys.append((heads[i % 2], int(t)))
    keys = np.array(keys, dtype=np.int64)
    rk, rv = oracle.sta_backward_dkdv(qc, kc, vc, doc, w.latent, w.tile, wins, w.softmax_scale, keys=keys)
    compare_grad(rows_of(dk, keys), rk, keys[:, 0], what="dk 720p")
    compare_grad(rows_of(dv, keys), rv, keys[:, 0], what="dv 720p")


def test_backward_mixed_windows_sampled(sta):
    w = sta_inputs.WORKLOADS[3]
    wins = sta_inputs.windows(w).tolist()
    # one head of each distinct window
    heads = sorted({tuple(x): h for h, x in reversed(list(enumerate(wins)))}.values())
    q, k, v = sta_inputs.make_qkv(w, device="cuda")
    do = sta_inputs.make_dout(w, device="cuda")
    plan, dq, dk, dv = gpu_grads(sta, q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    qc, kc, vc, doc = (x.cpu() for x in (q, k, v, do))
    toks = tile_rows(w.latent, w.tile, sample_tiles(w.latent, w.tile, 2, seed=8), 3, seed=9)
    rows = np.array([(h, t) for h in heads for t in toks], dtype=np.int64)
    ref = oracle.sta_backward_dq(qc, kc, vc, doc, w.latent, w.tile, wins, w.softmax_scale, rows=rows)
    compare_grad(rows_of(dq, rows), ref, rows[:, 0], what="dq mixed")
    small = [h for h in heads if tuple(wins[h]) == tuple(sta_inputs.W_SMALL)]
    if small:
        tt = oracle.tile_tokens(w.latent, w.tile, 7)
        keys = np.array([(small[0], int(t)) for t in tt[[0, 5, 200, 383]]], dtype=np.int64)
        rk, rv = oracle.sta_backward_dkdv(qc, kc, vc, doc, w.latent, w.tile, wins, w.softmax_scale, keys=keys)
        compare_grad(rows_of(dk, keys), rk, keys[:, 0], what="dk mixed")
        compare_grad(rows_of(dv, keys), rv, keys[:, 0], what="dv mixed")


def test_backward_large_scaled_heads_sampled_dq(sta):
    """The large workload (B=2, heads scaled by f_h in [0.5, 2]): dQ on sampled
    rows of two heads with different factors."""
    w = sta_inputs.WORKLOADS[5]
    q, k, v = sta_inputs.make_qkv(w, device="cuda")
    do = sta_inputs.make_dout(w, device="cuda")
    wins = sta_inputs.windows(w).tolist()
    f = sta_inputs.head_factors(w)
    h_lo, h_hi = int(torch.argmin(f)), int(torch.argmax(f))
    plan, dq, dk, dv = gpu_grads(sta, q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    qc, kc, vc, doc = (x.cpu() for x in (q, k, v, do))
    toks = tile_rows(w.latent, w.tile, sample_tiles(w.latent, w.tile, 1, seed=10), 2, seed=11)
    rows = np.array([(bh, t) for bh in (h_lo, w.heads + h_hi) for t in toks], dtype=np.int64)
    ref = oracle.sta_backward_dq(qc, kc, vc, doc, w.latent, w.tile, wins, w.softmax_scale, rows=rows)
    compare_grad(rows_of(dq, rows), ref, rows[:, 0], what="dq large")


def test_backward_deterministic_and_tile_major_entry(sta):
    """Two calls give the same bits (no atomics), and sta_backward on
    tile-major tensors equals the raster chain permuted."""
    latent, tile, B, H, d = (12, 16, 24), (6, 8, 8), 1, 2, 128
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(77)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
    windows = [[6, 8, 8], [12, 16, 16]]
    plan = sta.sta_plan(latent, tile, B, H, windows)
    scale = 1.0 / np.sqrt(d)
    o, lse = sta.sta_attention(q, k, v, plan, scale)
    a = sta.sta_attention_backward(q, k, v, o, lse, do, plan, scale)
    b = sta.sta_attention_backward(q, k, v, o, lse, do, plan, scale)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    tm = [torch.empty_like(x) for x in (q, k, v, o, do)]
    for x, y in zip((q, k, v, o, do), tm):
        sta.sta_tile_reorder(x, y, latent, tile)
    lt = torch.empty_like(lse)
    sta.sta_tile_reorder(lse, lt, latent, tile)
    ws = torch.empty(2 * B * H * N, dtype=torch.float32, device="cuda")
    dq, dk, dv = sta.sta_backward(plan, tm[0], tm[1], tm[2], tm[3], lt, tm[4], scale, workspace=ws)
    for x, ref in zip((dq, dk, dv), a):
        back = torch.empty_like(x)
        sta.sta_tile_unreorder(x, back, latent, tile)
        assert torch.equal(back, ref)
    # workspace plane 0 holds -D = -(dO . O) per tile-major row
    dref = (tm[4].float() * tm[3].float()).sum(-1).reshape(-1)
    torch.testing.assert_close(ws[: B * H * N], -dref, rtol=1e-5, atol=1e-5)
    assert sta.sta_last_device_status(plan) == 0


@pytest.mark.parametrize("latent,tile,d", [((30, 48, 80), (6, 8, 8), 128), ((12, 16, 16), (4, 8, 8), 128),
                                            ((18, 24, 24), (6, 8, 8), 64), ((8, 16, 16), (2, 8, 8), 128)])
def test_fused_raster_backward_equals_chain(sta, latent, tile, d):
    """sta_backward_raster gives the same bits as reorder -> sta_backward ->
    unreorder, on the 720p workload shape (2 heads) and smaller geometries."""
    B, H = 1, 2
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator(device="cuda").manual_seed(N + d)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g, device="cuda").to(torch.bfloat16) for _ in range(4))
    windows = [[3 * t for t in tile], list(tile)]
    plan = sta.sta_plan(latent, tile, B, H, windows)
    scale = 1.0 / np.sqrt(d)
    o, lse = sta.sta_attention(q, k, v, plan, scale)
    fused = sta.sta_attention_backward(q, k, v, o, lse, do, plan, scale)
    chain = sta.sta_attention_backward(q, k, v, o, lse, do, plan, scale, fused=False)
    for a, b in zip(fused, chain):
        assert torch.equal(a, b)
    assert sta.sta_last_device_status(plan) == 0


def test_autograd_function(sta):
    """StaAttention.apply inside autograd gives the same gradients as the
    explicit backward call."""
    latent, tile, B, H, d = (12, 16, 16), (6, 8, 8), 1, 2, 64
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(78)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
    plan = sta.sta_plan(latent, tile, B, H, [[6, 8, 8]] * H)
    qa, ka, va = (x.clone().requires_grad_(True) for x in (q, k, v))
    o = sta.StaAttention.apply(qa, ka, va, plan, 0.125)
    o.backward(do)
    o2, lse = sta.sta_attention(q, k, v, plan, 0.125)
    assert torch.equal(o.detach(), o2)
    ref = sta.sta_attention_backward(q, k, v, o2, lse, do, plan, 0.125)
    for got, r in zip((qa.grad, ka.grad, va.grad), ref):
        assert torch.equal(got, r)


def test_calls_from_a_fresh_thread(sta):
    """Forward and backward from a thread that has made no CUDA call before
    (as autograd's worker threads and thread pools are)."""
    import threading
    latent, tile, B, H, d = (12, 16, 16), (6, 8, 8), 1, 2, 64
    N = latent[0] * latent[1] * latent[2]
    g = torch.Generator().manual_seed(79)
    q, k, v, do = (torch.randn(B, H, N, d, generator=g).to(torch.bfloat16).cuda() for _ in range(4))
    plan = sta.sta_plan(latent, tile, B, H, [[6, 8, 8]] * H)
    o_ref, l_ref = sta.sta_attention(q, k, v, plan, 0.125)
    ref = sta.sta_attention_backward(q, k, v, o_ref, l_ref, do, plan, 0.125)
    torch.cuda.synchronize()
    box = {}

    def work():
        try:
            o, l = sta.sta_attention(q, k, v, plan, 0.125)
            box["fwd"] = (o, l)
            box["bwd"] = sta.sta_attention_backward(q, k, v, o, l, do, plan, 0.125)
            torch.cuda.synchronize()
        except Exception as e:  # reported below
            box["err"] = e

    t = threading.Thread(target=work)
    t.start()
    t.join()
    assert "err" not in box, box.get("err")
    assert torch.equal(box["fwd"][0], o_ref) and torch.equal(box["fwd"][1], l_ref)
    for a, b in zip(box["bwd"], ref):
        assert torch.equal(a, b)


@pytest.mark.parametrize("idx", [2, 4, 5])
def test_backward_full_size_invariants(sta, idx):
    """At every workload's full size: sum over keys of dV equals sum over
    queries of dO (each row of P sums to 1), and sum over keys of dK is ~0
    (each row of dS sums to 0).  Both hold at any size, so they cover dK and dV
    where the oracle cannot go.  Tolerances: the sums run over N rows whose
    terms carry bf16 rounding (relative 2^-9, random sign), so they are
    bounded against sqrt(sum of squares) of the summed terms: 2e-2 of it for
    dV, and for dK 2e-2 of sqrt(N) rms(dK).  For dK the rounding of dS to bf16
    (the operand of the dS^T Q product) and of O (inside D) dominates: an
    fp64 emulation of exactly those two roundings on N(0, 1) inputs, d = 128,
    1536 keys per query, gives a ratio of 6.7e-3 median and 1.0e-2 at the
    worst of 24 heads, so the bound leaves about 2x.  A missing or wrong D
    term leaves each row of dS summing to D_i instead of 0: an O(1) ratio."""
    w = sta_inputs.WORKLOADS[idx]
    q, k, v = sta_inputs.make_qkv(w, device="cuda")
    do = sta_inputs.make_dout(w, device="cuda")
    wins = sta_inputs.windows(w).tolist()
    plan, dq, dk, dv = gpu_grads(sta, q, k, v, do, w.latent, w.tile, wins, w.softmax_scale)
    for t in (dq, dk, dv):
        assert bool(torch.isfinite(t).all())
    dv_sum = dv.double().sum(dim=2)
    do_sum = do.double().sum(dim=2)
    do_norm = do.double().pow(2).sum(dim=2).sqrt()
    r_dv = float(((dv_sum - do_sum).abs() / do_norm).max())
    assert r_dv <= 2e-2, ("sum dV - sum dO", r_dv)
    dk_sum = dk.double().sum(dim=2)
    n = dk.shape[2]
    dk_scale = dk.double().pow(2).mean(dim=(2, 3)).sqrt().unsqueeze(-1) * n ** 0.5
    r_dk = float((dk_sum.abs() / dk_scale).max())
    assert r_dk <= 2e-2, ("sum dK", r_dk)
    print(f"workload {idx}: sum dV vs dO {r_dv:.2e}, sum dK {r_dk:.2e}")
    if idx == 4:
        # the full-window workload: dQ on sampled rows against the oracle
        toks = tile_rows(w.latent, w.tile, sample_tiles(w.latent, w.tile, 1, seed=14), 2, seed=15)
        rows = np.array([(h, t) for h in (0, 11) for t in toks], dtype=np.int64)
        ref = oracle.sta_backward_dq(q.cpu(), k.cpu(), v.cpu(), do.cpu(), w.latent, w.tile, wins,
                                     w.softmax_scale, rows=rows)
        compare_grad(rows_of(dq, rows), ref, rows[:, 0], what="dq full window")
