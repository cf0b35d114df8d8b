"""GPU parity of the window-search statistics (attention recall and output
error against full attention, per head) with the fp64 oracle.

Tolerances: recall, relative 1e-3 (the forward's LSE is fp32 arithmetic with
errors near 1e-6 relative; exp of an LSE difference turns an absolute LSE
error into the same relative recall error).  Output error: with eps =
2^-9 (rms(O_window) + rms(O_full)), the bf16 rounding of both outputs moves
the mean squared difference by at most 2 sqrt(mse) eps + eps^2.
"""
import numpy as np
import pytest
import torch

import oracle
import sta_inputs
from parity_util import sample_tiles, tile_rows

pytestmark = pytest.mark.gpu

RECALL_RTOL = 1e-3


@pytest.fixture(scope="module")
def sta():
    if not torch.cuda.is_available():
        pytest.fail("CUDA device required for -m gpu tests")
    import sparse_attention_video_sta_b200 as s
    return s


def mse_bound(mse_ref, o_w_ref, o_f_ref):
    eps = 2.0 ** -9 * (np.sqrt(np.mean(o_w_ref ** 2)) + np.sqrt(np.mean(o_f_ref ** 2)))
    return 2.0 * np.sqrt(mse_ref) * eps + eps * eps


def test_search_tiny_workload(sta):
    w = sta_inputs.WORKLOADS[1]
    q, k, v = sta_inputs.make_qkv(w)
    cands = [(6, 8, 8), (12, 16, 16), w.latent]
    res = sta.sta_window_search(q.cuda(), k.cuda(), v.cuda(), w.latent, w.tile, cands, w.softmax_scale)
    o_f, _ = oracle.sta_attention(q, k, v, w.latent, w.tile, [w.latent] * w.heads, w.softmax_scale)
    ref_mse = []
    for ci, c in enumerate(cands):
        rec = oracle.window_recall(q, k, w.latent, w.tile, [c] * w.heads, w.softmax_scale)
        o_c, _ = oracle.sta_attention(q, k, v, w.latent, w.tile, [c] * w.heads, w.softmax_scale)
        for h in range(w.heads):
            r_ref = rec[:, h].mean()
            assert abs(res["recall"][ci, h] - r_ref) <= RECALL_RTOL * r_ref, (c, h, res["recall"][ci, h], r_ref)
            m_ref = np.mean((o_c[:, h] - o_f[:, h]) ** 2)
            bound = mse_bound(m_ref, o_c[:, h], o_f[:, h])
            assert abs(res["mse"][ci, h] - m_ref) <= bound, (c, h, res["mse"][ci, h], m_ref, bound)
        ref_mse.append([np.mean((o_c[:, h] - o_f[:, h]) ** 2) for h in range(w.heads)])
    # the full window against itself
    assert np.all(res["recall"][2] == 1.0) and np.all(res["mse"][2] == 0.0)
    # the pick: a bound between the two sparse candidates' errors picks the larger window
    ref_mse = np.array(ref_mse)
    bound = float(np.sqrt(ref_mse[0].min() * ref_mse[1].max()))
    if ref_mse[1].max() < bound < ref_mse[0].min():
        pick = sta.sta_window_search(q.cuda(), k.cuda(), v.cuda(), w.latent, w.tile, cands, w.softmax_scale,
                                     max_mse=bound)
        assert pick["windows"] == [list(cands[1])] * w.heads
    pick = sta.sta_window_search(q.cuda(), k.cuda(), v.cuda(), w.latent, w.tile, cands, w.softmax_scale,
                                 min_recall=0.0)
    assert pick["windows"] == [list(cands[0])] * w.heads


def test_recall_720p_sampled_rows(sta):
    """Per-row recall exp(LSE_w - LSE_full) from the GPU forward against the
    oracle's definition on sampled rows, and the per-head reduction against a
    plain torch mean of the same GPU values."""
    w = sta_inputs.WORKLOADS[2]
    q, k, v = sta_inputs.make_qkv(w, device="cuda")
    B, H = w.batch, w.heads
    full = sta.sta_plan(w.latent, w.tile, B, H, [w.latent] * H)
    plan = sta.sta_plan(w.latent, w.tile, B, H, [sta_inputs.W_SMALL] * H)
    o_f, l_f = sta.sta_attention(q, k, v, full, w.softmax_scale)
    o_w, l_w = sta.sta_attention(q, k, v, plan, w.softmax_scale)
    rec_gpu = torch.exp(l_w.double() - l_f.double())
    recall, mse = sta.sta_window_stats(l_w, l_f, o_w, o_f)
    torch.testing.assert_close(recall, rec_gpu.mean(dim=2), rtol=1e-6, atol=0)
    torch.testing.assert_close(mse, ((o_w.double() - o_f.double()) ** 2).mean(dim=(2, 3)), rtol=1e-5, atol=0)
    heads = [0, 17]
    toks = tile_rows(w.latent, w.tile, sample_tiles(w.latent, w.tile, 2, seed=12), 4, seed=13)
    rows = np.array([(h, t) for h in heads for t in toks], dtype=np.int64)
    ref = oracle.window_recall(q.cpu(), k.cpu(), w.latent, w.tile, [sta_inputs.W_SMALL] * H, w.softmax_scale,
                               rows=rows)
    got = rec_gpu.reshape(-1, w.tokens)[rows[:, 0], rows[:, 1]].cpu().numpy()
    np.testing.assert_allclose(got, ref, rtol=RECALL_RTOL, atol=0)
    assert sta.sta_last_device_status(plan) == 0 and sta.sta_last_device_status(full) == 0
