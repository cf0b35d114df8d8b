"""The per-head window pick (sta_window_pick, host only) against its rule.

Rule (the library's reading; the pages profile candidate windows per head but
give no selection rule): each head takes the candidate with the fewest
attended tiles, ties to the one listed first, whose recall is at least
``min_recall`` and whose output error at most ``max_mse`` (each bound
optional); the window covering the volume when none qualifies.  CPU only.
"""
import math

import numpy as np
import pytest

import sparse_attention_video_sta_b200 as sta


def rule(latent, tile, cands, recall, mse, max_mse, min_recall):
    n = [-(-latent[i] // tile[i]) for i in range(3)]
    tiles = [math.prod(min(c[i] // tile[i], n[i]) for i in range(3)) for c in cands]
    order = sorted(range(len(cands)), key=lambda i: (tiles[i], i))
    out = []
    for h in range(recall.shape[1] if len(cands) else 1):
        pick = list(latent)
        for i in order:
            if (max_mse is None or mse[i, h] <= max_mse) and (min_recall is None or recall[i, h] >= min_recall):
                pick = list(cands[i])
                break
        out.append(pick)
    return out


@pytest.mark.parametrize("seed", range(6))
def test_pick_matches_rule_on_random_stats(seed):
    rng = np.random.default_rng(seed)
    latent, tile, H = (30, 48, 80), (6, 8, 8), 7
    pool = [(6, 8, 8), (18, 24, 24), (30, 40, 40), (12, 16, 24), (24, 16, 16), (30, 48, 80), (60, 96, 160)]
    cands = [pool[i] for i in rng.choice(len(pool), size=5, replace=False)]
    recall = rng.uniform(0, 1, (len(cands), H))
    mse = rng.uniform(0, 1e-3, (len(cands), H))
    for max_mse, min_recall in ((None, None), (5e-4, None), (None, 0.5), (2e-4, 0.7), (0.0, 1.0)):
        got = sta.sta_window_pick(latent, tile, H, cands, recall, mse, max_mse, min_recall)
        assert got == rule(latent, tile, cands, recall, mse, max_mse, min_recall)


def test_pick_edge_cases():
    latent, tile = (13, 21, 18), (6, 8, 8)   # padded: 3 x 3 x 3 tiles
    # equal tile counts: the first listed wins; a window wider than the volume
    # counts as the volume
    cands = [(12, 16, 16), (12, 16, 16), (60, 64, 64)]
    r = np.ones((3, 2))
    m = np.zeros((3, 2))
    assert sta.sta_window_pick(latent, tile, 2, cands, r, m) == [[12, 16, 16]] * 2
    # nothing qualifies: the volume
    assert sta.sta_window_pick(latent, tile, 2, cands, r * 0.1, m, None, 0.5) == [list(latent)] * 2
    # no candidates at all
    assert sta.sta_window_pick(latent, tile, 3, [], None, None) == [list(latent)] * 3
    # a candidate that is not a tile multiple is rejected
    with pytest.raises(sta.StaError):
        sta.sta_window_pick(latent, tile, 2, [(7, 8, 8)], r[:1], m[:1])
