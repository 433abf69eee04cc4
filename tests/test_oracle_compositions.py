"""Pins of the oracle's whole-path compositions (``oracle/pipeline.py``).

The stage functions are pinned in ``test_oracle_pins.py``; here the decode
compositions are checked on inputs built so that every intermediate is known
by hand: which entries the compressor produces, which ones the indexer ranks
first (ties included), which raw rows form the window and what attention over
them returns.  Each pin is then run against copies of the composition with a
plausible mistake planted in its source text (wrong window tensor or offset,
the new entry off by one, the c4a overlap switched on for c128a, a branch
swap, ...), and must reject every one of them.

Sources: "DeepSeek V4 结构速览", sections "核心设计" item 2 (c4a / c128a
geometry, k among the visible entries, the 128-token raw window), "CSA（c4a
路线）" (selected entries concatenated with the window, K = V), "HCA（c128a
路线）" (dense over every entry, sink) and "C4A Compressor" (the previous
block comes from the second branch).
"""

import inspect
import math
import textwrap

import numpy as np
import pytest

from oracle import csa, pipeline


def mutant(fn, old, new):
    """A copy of ``fn`` whose source has ``old`` replaced by ``new`` (which must occur)."""
    src = textwrap.dedent(inspect.getsource(fn))
    assert old in src, old
    ns = dict(fn.__globals__)
    exec(compile(src.replace(old, new), "<mutant of %s>" % fn.__name__, "exec"), ns)
    return ns[fn.__name__]


# ---------------------------------------------------------------------------
# HCA decode: c128a geometry (m = 128, no previous block), dense attention
# ---------------------------------------------------------------------------

HCA = dict(m=128, L=4 * 128, c=8, n_w=16)


def _hca_inputs(seed=11):
    """Raw rows whose block means are known unit-rms vectors, and uniform pooling weights.

    Block i of C_a is v_i (entries +-1, so unit rms and exact in float32) plus a
    pattern that sums to zero over the block, so the per-channel softmax of equal
    logits (Z_a = 0, B_a = 0) pools v_i.  C_b / Z_b / B_b carry unrelated values
    that c128a must never read.
    """
    m, L, c = HCA["m"], HCA["L"], HCA["c"]
    E = L // m
    rng = np.random.default_rng(seed)
    v = rng.choice([-1.0, 1.0], size=(E, c))
    pat = rng.normal(size=(m, c))
    pat -= pat.mean(axis=0)
    C_a = np.concatenate([v[i] + pat for i in range(E)], axis=0)
    main = dict(C_a=C_a, Z_a=np.zeros((L, c)), B_a=np.zeros((m, c)),
                C_b=rng.normal(size=(L, c)) * 3.0, Z_b=rng.normal(size=(L, c)),
                B_b=rng.normal(size=(m, c)))
    return main, v


def hca_pin(fn):
    """Check an HCA decode composition ``fn`` (signature of ``pipeline.hca_decode_seq``)."""
    m, L, c, n_w = HCA["m"], HCA["L"], HCA["c"], HCA["n_w"]
    E = L // m
    t = L - 1
    main, v = _hca_inputs()
    sink = np.array([0.25, -1.5])
    kw = dict(L=L, m=m, d_rope=0, theta=1e4, eps=0.0, n_w=n_w, scale=0.125, kv_dtype="f32")
    # (1) q = 0: every logit is 0, so o = (sum of the E entries + the window rows) / (e^sink + E + n_w)
    r = fn(main, np.zeros((2, c)), sink, **kw)
    assert r["kv"].shape == (E, c)
    np.testing.assert_allclose(r["kv"], v, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["new_entry"], v[E - 1], rtol=0, atol=1e-12)
    rows_sum = v.sum(axis=0) + main["C_a"][t - n_w + 1:t + 1].sum(axis=0)
    for h in range(2):
        den = math.exp(sink[h]) + E + n_w
        np.testing.assert_allclose(r["out_f64"][h], rows_sum / den, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["lse"][h], math.log(den), rtol=1e-13)
    # (2) random q: the same as CSA attention with top-k = every visible entry, over the
    #     entries compressed one by one without overlap (HCA equals CSA with k = E)
    rng = np.random.default_rng(5)
    q = rng.normal(size=(2, c)) * 4.0
    r = fn(main, q, sink, **kw)
    kv = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], None, None, None, m, False,
                              np.arange(E), 0, 1e4, 0.0)
    scores = rng.normal(size=(1, E))
    idx, cnt = csa.topk(scores, np.array([t]), m, E)
    assert int(cnt[0]) == E
    o, lse = csa.sparse_attn(q[None], pipeline.round_out(kv, "f32"), idx, cnt, main["C_a"],
                             np.array([t]), sink, n_w, 0.125)
    np.testing.assert_allclose(r["out_f64"], o[0], rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(r["lse"], lse[0], rtol=1e-13)


def test_hca_decode_composition_closed_form():
    hca_pin(pipeline.hca_decode_seq)


@pytest.mark.parametrize("old,new", [
    ('main["C_a"][csa.window_rows', 'main["C_b"][csa.window_rows'),        # window tensor
    ("csa.window_rows(t, n_w)", "csa.window_rows(t - 1, n_w)"),            # window offset
    ("csa.window_rows(t, n_w)", "csa.window_rows(t, n_w - 1)"),            # window length
    ("t = L - 1", "t = L - 2"),                                            # query position
    ("None, None, None, m, False", 'main["C_b"], main["Z_b"], main["B_b"], m, True'),  # c4a overlap
    ("m, False,\n                            0, E,", "m, False,\n                            0, E - 1,"),  # entry count
    ("new_entry=kv[E - 1]", "new_entry=kv[E - 2]"),                        # the entry the step completes
    ("csa.attend(np.asarray(q), rows, sink, scale)", "csa.attend(np.asarray(q), rows, sink, 1.0)"),
])
def test_hca_pin_rejects_planted_mistakes(old, new):
    bad = mutant(pipeline.hca_decode_seq, old, new)
    with pytest.raises(Exception):
        hca_pin(bad)


# ---------------------------------------------------------------------------
# CSA decode: c4a geometry (m = 4, overlapped), FP8 indexer, top-k, window
# ---------------------------------------------------------------------------

CSA_G = dict(m=4, L=64, c=8, cI=8, n_w=6, k=3)
# index query on the E4M3 grid with amax 448 (scale exactly 1), distinct per channel
Q_INDEX = np.array([448.0, 416.0, 384.0, 352.0, 320.0, 288.0, 256.0, 240.0])


def _block_const_branch(vecs, tail, m, rng):
    """A branch whose pooled entry i is exactly vecs[i] whatever the softmax weights.

    Entry i pools rows [m(i-1), mi) of C_b and [mi, mi+m) of C_a, so C_a's block j
    holds vecs[j] and C_b's block j holds vecs[j+1] (the last C_b block holds
    ``tail``, which no entry reads).  Logits and biases are random.
    """
    E, c = vecs.shape
    C_a = np.repeat(vecs, m, axis=0)
    C_b = np.repeat(np.concatenate([vecs[1:], tail[None]], axis=0), m, axis=0)
    n = E * m
    return dict(C_a=C_a, C_b=C_b, Z_a=rng.normal(size=(n, c)), Z_b=rng.normal(size=(n, c)),
                B_a=rng.normal(0, 0.5, (m, c)), B_b=rng.normal(0, 0.5, (m, c)))


def _csa_inputs(seed=3):
    m, L, c, cI = CSA_G["m"], CSA_G["L"], CSA_G["c"], CSA_G["cI"]
    E = L // m
    rng = np.random.default_rng(seed)
    v = rng.choice([-1.0, 1.0], size=(E, c))                 # unit rms latent entries
    u = np.zeros((E, cI))
    u[np.arange(E), np.arange(E) % cI] = math.sqrt(cI)       # one-hot index keys of unit rms
    main = _block_const_branch(v, rng.choice([-1.0, 1.0], size=c) * 2.0, m, rng)
    index = _block_const_branch(u, np.full(cI, 1.0), m, rng)
    return main, index, v, u


def csa_pin(fn):
    """Check a CSA decode composition ``fn`` (signature of ``pipeline.csa_decode_seq``)."""
    m, L, c, n_w, k = CSA_G["m"], CSA_G["L"], CSA_G["c"], CSA_G["n_w"], CSA_G["k"]
    E = L // m
    t = L - 1
    main, index, v, u = _csa_inputs()
    sink = np.array([0.5, -0.75])
    w = np.array([0.5])
    kw = dict(L=L, m=m, d_rope=0, theta=1e4, eps=0.0, k=k, n_w=n_w, scale=0.125,
              kv_dtype="f32", idx_dtype="fp8")
    r = fn(main, index, np.zeros((2, c)), Q_INDEX[None], w, sink, **kw)
    # keys: entry s is one-hot on channel s % 8; the FP8 row code is 448 on it
    np.testing.assert_allclose(r["kI"], u, rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["new_kI"], u[E - 1], rtol=0, atol=1e-12)
    # scores: 0.5 * q[s % 8] * sqrt(8): entries s and s + 8 tie, ties go to the lower s,
    # so the top 3 are 0 and 8 (channel 0) and 1 (channel 1, before 9)
    ks = np.float32(np.float32(math.sqrt(8)) / np.float32(448.0))
    expect = 0.5 * Q_INDEX[np.arange(E) % 8] * 448.0 * float(ks)
    np.testing.assert_allclose(r["scores"], expect, rtol=2 ** -8)
    assert r["cnt"] == k
    np.testing.assert_array_equal(r["idx"], [0, 1, 8])
    np.testing.assert_allclose(r["new_entry"], v[E - 1], rtol=0, atol=1e-12)
    np.testing.assert_allclose(r["kv_sel"], v[[0, 1, 8]], rtol=0, atol=1e-12)
    # q = 0: o = (v_0 + v_1 + v_8 + the window rows of C_a) / (e^sink + k + n_w); the window
    # rows t-5..t are blocks 14 (two rows) and 15 (four rows) of C_a
    rows_sum = v[0] + v[1] + v[8] + 2 * v[14] + 4 * v[15]
    for h in range(2):
        den = math.exp(sink[h]) + k + n_w
        np.testing.assert_allclose(r["out_f64"][h], rows_sum / den, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(r["lse"][h], math.log(den), rtol=1e-13)


def test_csa_decode_composition_closed_form():
    csa_pin(pipeline.csa_decode_seq)


@pytest.mark.parametrize("old,new", [
    ('main["C_a"][csa.window_rows', 'main["C_b"][csa.window_rows'),        # window tensor
    ("csa.window_rows(t, n_w)", "csa.window_rows(t - 1, n_w)"),            # window offset
    ("t = L - 1", "t = L - 2"),                                            # query position
    ("[E - 1], d_rope, theta, eps)[0]", "[E - 2], d_rope, theta, eps)[0]"),  # new entry
    ("new_kI=kI[E - 1]", "new_kI=kI[E - 2]"),
    ('index["C_a"], index["Z_a"], index["B_a"], index["C_b"], index["Z_b"],\n'
     '                            index["B_b"]',
     'index["C_b"], index["Z_b"], index["B_b"], index["C_a"], index["Z_a"],\n'
     '                            index["B_a"]'),                          # index branches swapped
    ("idx, cnt = csa.topk(scores, np.array([t]), m, k)",
     "idx, cnt = csa.topk(scores, np.array([t]), m, k + 1)"),              # selection size
    ("sel = idx[0, :cnt[0]].astype", "sel = (idx[0, :cnt[0]] + 1).astype"),  # selection offset
    ("np.asarray(w)[None]", "np.asarray(w)[None] * 0.0"),                  # head weights dropped
])
def test_csa_pin_rejects_planted_mistakes(old, new):
    bad = mutant(pipeline.csa_decode_seq, old, new)
    with pytest.raises(Exception):
        csa_pin(bad)


# ---------------------------------------------------------------------------
# decode at any position (variable-length batches, paged state)
# ---------------------------------------------------------------------------

def _rand_inputs(n, c, cI, H, HI, m, seed):
    rng = np.random.default_rng(seed)
    br = lambda cc: dict(C_a=rng.normal(size=(n, cc)), Z_a=rng.normal(size=(n, cc)),  # noqa: E731
                         B_a=rng.normal(0, 0.5, (m, cc)), C_b=rng.normal(size=(n, cc)),
                         Z_b=rng.normal(size=(n, cc)), B_b=rng.normal(0, 0.5, (m, cc)))
    return (br(c), br(cI), rng.normal(size=(n, H, c)), rng.normal(size=(n, HI, cI)),
            rng.uniform(size=(n, HI)) / 4, rng.normal(size=H))


def test_decode_at_any_position_equals_the_prefill_row():
    n, m, c, cI, H, HI = 96, 4, 16, 8, 2, 2
    main, index, q, qI, w, sink = _rand_inputs(n, c, cI, H, HI, m, 21)
    kw = dict(m=m, d_rope=4, theta=1e4, eps=1e-6, k=5, n_w=6, scale=0.25, kv_dtype="f32",
              idx_dtype="fp8")
    pre = pipeline.csa_prefill(main, index, q, qI, w, sink, score_dtype="bf16", **kw)
    for t in (0, 1, 2, 3, 4, 5, 22, 23, 24, 37, 63, 94, 95):
        d = pipeline.csa_decode_at(main, index, q[t], qI[t], w[t], sink, t=t, **kw)
        np.testing.assert_array_equal(d["idx"], pre["idx"][t])
        np.testing.assert_allclose(d["out_f64"], pre["out_f64"][t], rtol=1e-12, atol=1e-14)
        if (t + 1) % m == 0:
            np.testing.assert_allclose(d["new_entry"], pre["kv"][(t + 1) // m - 1], rtol=1e-13)
        else:
            assert d["new_entry"] is None
    # the block-completing last token is the whole-sequence decode step
    L = n
    full = pipeline.csa_decode_seq(main, index, q[L - 1], qI[L - 1], w[L - 1], sink, L=L, **kw)
    at = pipeline.csa_decode_at(main, index, q[L - 1], qI[L - 1], w[L - 1], sink, t=L - 1, **kw)
    np.testing.assert_allclose(at["out_f64"], full["out_f64"], rtol=1e-13)


def test_decode_at_reads_nothing_after_t():
    n, m, c, cI, H, HI = 64, 4, 8, 8, 2, 1
    main, index, q, qI, w, sink = _rand_inputs(n, c, cI, H, HI, m, 22)
    kw = dict(m=m, d_rope=2, theta=1e4, eps=1e-6, k=3, n_w=4, scale=0.3, kv_dtype="f32",
              idx_dtype="f32")
    t = 29
    a = pipeline.csa_decode_at(main, index, q[t], qI[t], w[t], sink, t=t, **kw)
    for br in (main, index):
        for name in ("C_a", "Z_a", "C_b", "Z_b"):
            br[name][t + 1:] = 1e3
    b = pipeline.csa_decode_at(main, index, q[t], qI[t], w[t], sink, t=t, **kw)
    np.testing.assert_array_equal(a["out_f64"], b["out_f64"])


def test_hca_decode_at_any_position():
    n, m, c, H = 4 * 16, 16, 8, 2
    main, _, q, _, _, sink = _rand_inputs(n, c, 8, H, 1, m, 23)
    kw = dict(m=m, d_rope=2, theta=1e4, eps=0.0, n_w=5, scale=0.3, kv_dtype="f32")
    kv_all = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], None, None, None, m, False,
                                  np.arange(n // m), 2, 1e4, 0.0)
    for t in (0, 14, 15, 16, 40, 63):
        r = pipeline.hca_decode_at(main, q[t], sink, t=t, **kw)
        o, _ = csa.dense_attn(q[t:t + 1], pipeline.round_out(kv_all, "f32"), main["C_a"], [t],
                              sink, 5, 0.3, m)
        np.testing.assert_allclose(r["out_f64"], o[0], rtol=1e-12, atol=1e-14)
    full = pipeline.hca_decode_seq(main, q[n - 1], sink, L=n, **kw)
    np.testing.assert_allclose(pipeline.hca_decode_at(main, q[n - 1], sink, t=n - 1, **kw)["out_f64"],
                               full["out_f64"], rtol=1e-13)
