"""Pins of the oracle's CSA2 pieces: the hierarchical (candidate-pool) indexer and the
Reuse / Reindex decode modes.

Source: "DeepSeek Technical Reports", section CSA2 (Cross-Layer KV and Index
Reuse: Reuse layers attend over an earlier layer's selection; Hierarchical
Sparse Indexer: a full indexer yields a larger candidate pool, later Reindex
layers score again with their own query, searching only that pool).
"""

import numpy as np
import pytest

from oracle import csa, pipeline

from test_oracle_compositions import _csa_inputs, mutant


def _tiny(T=5, E=40, H=3, d=8, seed=0):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(T, H, d))
    w = rng.uniform(size=(T, H))
    k = rng.normal(size=(E, d))
    return q, w, k, rng


def test_pool_of_every_visible_entry_is_the_full_indexer():
    m = 4
    q, w, kI, _ = _tiny()
    E = kI.shape[0]
    qpos = np.array([3, 50, 101, 158, 159])
    pool = np.tile(np.arange(E), (len(qpos), 1))
    for k in (1, 6, 40):
        ref = csa.topk(csa.index_scores(q, w, kI, qpos, m, "bf16"), qpos, m, k)
        got = csa.pool_topk(q, w, kI, pool, np.full(len(qpos), E), qpos, m, k)
        np.testing.assert_array_equal(got[0], ref[0])
        np.testing.assert_array_equal(got[1], ref[1])


def _brute(q, w, kI, pool_row, cnt, t, m, k):
    """Selection by a plain sort of (-score, entry) over the visible pool entries."""
    ev = (t + 1) // m
    full = csa.index_scores(q[None], w[None], kI, np.array([t]), m, "bf16")[0]
    cand = [int(e) for e in pool_row[:cnt] if 0 <= e < ev]
    best = sorted(cand, key=lambda e: (-full[e], e))[:k]
    return sorted(best)


def test_pool_topk_equals_brute_force_with_ties_and_causality():
    m = 4
    q, w, kI, rng = _tiny(T=6, E=64, seed=3)
    kI[10] = kI[20]                      # equal keys: equal scores, the lower entry first
    kI[33] = kI[20]
    qpos = np.array([255, 255, 100, 40, 7, 3])
    P = 24
    pool = np.full((6, P), -1, dtype=np.int64)
    cnt = np.zeros(6, dtype=np.int64)
    for r in range(6):
        c = np.sort(rng.choice(64, size=P - r, replace=False))
        c[:3] = [10, 20, 33] if r < 2 else c[:3]
        c = np.sort(np.unique(c))
        pool[r, :len(c)] = c
        cnt[r] = len(c)
    for k in (1, 2, 5, 30):
        idx, n = csa.pool_topk(q, w, kI, pool, cnt, qpos, m, k)
        for r in range(6):
            ref = _brute(q[r], w[r], kI, pool[r], cnt[r], qpos[r], m, k)
            assert n[r] == len(ref)
            assert list(idx[r, :n[r]]) == ref
            assert np.all(idx[r, n[r]:] == -1)


def test_pool_topk_all_tied_keeps_the_lowest_visible_entries():
    m = 4
    q, w, kI, rng = _tiny(T=2, E=50, seed=5)
    kI[:] = kI[0]                        # every score equal
    pool = np.array([[3, 9, 11, 17, 30, 41, -1, -1], [0, 2, 4, 6, 8, 10, 12, 14]])
    cnt = np.array([6, 8])
    qpos = np.array([4 * 20 - 1, 4 * 9 - 1])   # E(t) = 20 and 9
    idx, n = csa.pool_topk(q, w, kI, pool, cnt, qpos, m, 3)
    np.testing.assert_array_equal(idx, [[3, 9, 11], [0, 2, 4]])
    idx, n = csa.pool_topk(q, w, kI, pool, cnt, qpos, m, 6)
    np.testing.assert_array_equal(n, [4, 5])               # 30, 41 and 10.. are not visible
    np.testing.assert_array_equal(idx[1], [0, 2, 4, 6, 8, -1])


@pytest.mark.parametrize("old,new", [
    ("np.lexsort((cand, -sc))", "np.lexsort((-cand, -sc))"),          # tie-break flipped
    ("(cand < min(ev, k_I.shape[0]))", "(cand < k_I.shape[0])"),    # causality dropped
    ("np.maximum(dots, 0.0) @ w[r]", "dots @ w[r]"),                  # ReLU dropped
    ("keep = np.sort(cand[order[:min(k, len(cand))]])",
     "keep = cand[order[:min(k, len(cand))]]"),                       # output not ascending
])
def test_pool_topk_pins_reject_planted_mistakes(old, new):
    bad = mutant(csa.pool_topk, old, new)
    with pytest.raises(AssertionError):
        orig = csa.pool_topk
        try:
            csa.pool_topk = bad
            test_pool_topk_equals_brute_force_with_ties_and_causality()
            test_pool_of_every_visible_entry_is_the_full_indexer()
            test_pool_topk_all_tied_keeps_the_lowest_visible_entries()
        finally:
            csa.pool_topk = orig


def _decode(mode, **kw):
    from test_oracle_compositions import CSA_G
    m, L, n_w = CSA_G["m"], CSA_G["L"], CSA_G["n_w"]
    main, index, v, u = _csa_inputs()
    rng = np.random.default_rng(9)
    q = rng.normal(size=(2, CSA_G["c"]))
    qI = rng.normal(size=(3, CSA_G["cI"]))
    w = rng.uniform(size=3)
    sink = np.array([0.1, -0.2])
    return pipeline.csa_decode_seq(main, index, q, qI, w, sink, L=L, m=m, d_rope=4, theta=1e4,
                                   eps=1e-6, k=5, n_w=n_w, scale=0.3, kv_dtype="f32",
                                   idx_dtype="fp8", mode=mode, **kw)


def test_decode_modes_agree_with_the_full_path():
    full = _decode("full")
    E = 16
    # Reuse of this layer's own selection, and Reindex over every entry or over a pool that
    # holds the full top-k, all give the full path's result
    reuse = _decode("reuse", idx_in=full["idx"])
    every = _decode("reindex", pool=np.arange(E))
    top10 = csa.topk(full["scores"][None], np.array([63]), 4, 10)[0][0]
    pool = _decode("reindex", pool=top10)
    for r in (reuse, every, pool):
        np.testing.assert_array_equal(r["idx"], full["idx"])
        np.testing.assert_allclose(r["out_f64"], full["out_f64"], rtol=1e-13)
    # a pool that misses some of the full top-k keeps the best of what it has
    sub = np.setdiff1d(np.arange(E), full["idx"][:2])
    r = _decode("reindex", pool=sub)
    assert set(r["idx"][:r["cnt"]]) <= set(sub)
    assert not set(full["idx"][:2]) & set(r["idx"][:r["cnt"]])
    # Reuse attends exactly the given rows plus the window, whatever this layer's scores
    given = np.array([1, 7, 12, -1, -1])
    r = _decode("reuse", idx_in=given)
    assert r["cnt"] == 3
    np.testing.assert_array_equal(r["idx"][:3], [1, 7, 12])
