"""Pins of the oracle's attention recall (share of a row's full-attention
softmax mass inside its STA window) against facts other than its own code:

- q = 0 makes every score equal, so recall = |A_i| / N exactly, with |A_i|
  the clamped window volume in tokens (closed form);
- a window covering the volume gives recall 1;
- a dense fp64 softmax (scipy) summed over the brute-force nearest-centre
  mask of the forward pins (library routine + independent mask);
- nested windows give non-decreasing recall;
- recall = exp(LSE_window - LSE_full) with the (separately pinned) forward
  oracle's LSEs.
"""
import numpy as np
import pytest
import torch
from scipy.special import softmax

import oracle
from test_oracle_pins import brute_mask


def rand_bf16(seed, shape, scale=1.0):
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(shape, generator=g) * scale).to(torch.bfloat16)


def test_uniform_scores_closed_form():
    latent, tile, d = (6, 8, 12), (2, 4, 4), 8
    N = 6 * 8 * 12
    windows = [[2, 4, 4], [4, 8, 8], [6, 4, 12]]
    q = torch.zeros(1, 3, N, d, dtype=torch.bfloat16)
    k = rand_bf16(1, (1, 3, N, d))
    rec = oracle.window_recall(q, k, latent, tile, windows, 0.5)
    for h, w in enumerate(windows):
        e = [min(w[i] // tile[i], latent[i] // tile[i]) for i in range(3)]
        expect = e[0] * e[1] * e[2] * (tile[0] * tile[1] * tile[2]) / N
        np.testing.assert_allclose(rec[0, h], expect, rtol=1e-13, atol=0)


def test_full_window_is_one():
    latent, tile, d = (4, 8, 8), (2, 4, 4), 16
    N = 256
    q, k = rand_bf16(2, (2, 1, N, d), 2.0), rand_bf16(3, (2, 1, N, d))
    rec = oracle.window_recall(q, k, latent, tile, [[4, 8, 8]], 0.25)
    assert np.all(rec == 1.0)


@pytest.mark.parametrize("latent,tile,windows", [
    ((6, 8, 8), (2, 4, 4), [[2, 4, 4], [4, 8, 4], [6, 4, 8]]),
    ((4, 8, 12), (2, 4, 4), [[2, 8, 8], [4, 4, 4]]),
])
def test_matches_dense_softmax_with_brute_mask(latent, tile, windows):
    d = 8
    N = latent[0] * latent[1] * latent[2]
    H = len(windows)
    q, k = rand_bf16(4, (1, H, N, d), 1.5), rand_bf16(5, (1, H, N, d), 1.5)
    scale = 0.41
    rec = oracle.window_recall(q, k, latent, tile, windows, scale)
    s64 = float(np.float32(scale))
    for h, w in enumerate(windows):
        qq, kk = q[0, h].double().numpy(), k[0, h].double().numpy()
        p = softmax(s64 * (qq @ kk.T), axis=1)
        expect = (p * brute_mask(latent, tile, w)).sum(axis=1)
        np.testing.assert_allclose(rec[0, h], expect, rtol=1e-12, atol=1e-14)


def test_nested_windows_non_decreasing():
    latent, tile, d = (10, 10, 10), (2, 2, 2), 8
    N = 1000
    q, k = rand_bf16(6, (1, 1, N, d), 2.0), rand_bf16(7, (1, 1, N, d))
    prev = None
    for e in (1, 3, 5):
        rec = oracle.window_recall(q, k, latent, tile, [[2 * e] * 3], 0.35)
        if prev is not None:
            assert np.all(rec >= prev - 1e-15)
        prev = rec
    assert np.all(prev <= 1.0 + 1e-15)


def test_recall_is_lse_difference():
    latent, tile, d = (6, 8, 8), (2, 4, 4), 16
    N = 384
    q, k, v = rand_bf16(8, (1, 2, N, d), 1.5), rand_bf16(9, (1, 2, N, d), 1.5), rand_bf16(10, (1, 2, N, d))
    windows = [[2, 4, 4], [4, 4, 8]]
    rec = oracle.window_recall(q, k, latent, tile, windows, 0.3)
    _, lse_w = oracle.sta_attention(q, k, v, latent, tile, windows, 0.3)
    _, lse_f = oracle.sta_attention(q, k, v, latent, tile, [list(latent)] * 2, 0.3)
    np.testing.assert_allclose(rec, np.exp(lse_w - lse_f), rtol=1e-12)
