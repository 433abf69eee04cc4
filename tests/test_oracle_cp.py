"""Pin of the decomposition the context-parallel decode relies on, on the oracle's own
top-k: the k best entries of the whole cache are the k best among the shards' own k best
(order: score descending, entry ascending), with causal positions shifted per shard.
Brute force on small rows with heavy ties across the shard borders.

Source: "DeepSeek Technical Reports", section DSA (the top-k of a query's index scores).
"""

import numpy as np
import pytest

from oracle import csa


def _sharded(scores, t, m, k, bounds):
    cand_s, cand_e = [], []
    for e0, n in bounds:
        if (t + 1) // m <= e0:                             # nothing of this shard visible
            continue
        idx, cnt = csa.topk(scores[None, e0:e0 + n], np.array([t - m * e0]), m, k)
        sel = idx[0, :cnt[0]]
        cand_s += list(scores[e0 + sel])
        cand_e += list(e0 + sel)
    cand_s, cand_e = np.array(cand_s, dtype=np.float64), np.array(cand_e, dtype=np.int64)
    # top-k of the candidates; they are in ascending entry order, so position ties go to
    # the lower entry and every candidate is visible
    idx, cnt = csa.topk(cand_s[None], np.array([len(cand_s) - 1]), 1, k)
    return cand_e[idx[0, :cnt[0]]], int(cnt[0])


@pytest.mark.parametrize("seed", range(6))
@pytest.mark.parametrize("bounds", [[(0, 8), (8, 8)], [(0, 5), (5, 7), (12, 9)], [(0, 16), (16, 5)]])
def test_top_k_of_the_shards_top_k_is_the_global_top_k(seed, bounds):
    rng = np.random.default_rng(seed)
    E = bounds[-1][0] + bounds[-1][1]
    m = 4
    scores = np.round(rng.normal(size=E) * 2) / 2          # heavy ties
    for k in (1, 3, 7, E - 2):
        for t in (m * E - 1, m * (E // 2) + 1, m * 3):   # all, part, few entries visible
            ev = (t + 1) // m
            want, wc = csa.topk(scores[None], np.array([t]), m, k)
            got, gc = _sharded(scores, t, m, k, bounds)
            assert gc == wc[0] == min(k, ev)
            np.testing.assert_array_equal(got, want[0, :wc[0]])


def test_the_pin_rejects_a_wrong_tie_rule():
    # were the shards' candidates merged in reverse rank order, a tie across the border
    # would go to the higher entry: the check above must see that
    scores = np.zeros(16)
    want, _ = csa.topk(scores[None], np.array([4 * 16 - 1]), 4, 3)
    cand = [(8 + j, 0.0) for j in range(3)] + [(j, 0.0) for j in range(3)]   # reversed
    cs = np.array([s for _, s in cand])
    ce = np.array([e for e, _ in cand])
    idx, cnt = csa.topk(cs[None], np.array([len(cs) - 1]), 1, 3)
    assert not np.array_equal(ce[idx[0, :cnt[0]]], want[0, :3])
