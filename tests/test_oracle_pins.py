"""Pins of the CPU oracle against facts fixed outside it.

Each test checks the oracle against a closed form, a library routine for a
special case, an invariant of the definition, brute force on a tiny input, or
a value the pages print (``tests/golden``).  They are chosen so that a dropped
term, a wrong sign or index, a swapped branch or a transposed operand in the
oracle fails at least one of them.
"""

import json
import math
import os

import ml_dtypes
import numpy as np
import pytest
import scipy.special
import torch

from oracle import codecs, csa, pipeline

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


# ---------------------------------------------------------------------------
# number formats
# ---------------------------------------------------------------------------

def _finite_e4m3_values():
    codes = np.arange(256, dtype=np.uint8)
    vals = codecs.e4m3_decode(codes)
    keep = np.isfinite(vals)
    return codes[keep], vals[keep]


def test_e4m3_decode_table_fixed_points():
    # OCP E4M3FN: 448 largest finite, 2^-6 smallest normal, 2^-9 smallest subnormal, NaN at S.1111.111
    assert codecs.e4m3_decode(np.uint8(0x7E)) == 448.0
    assert codecs.e4m3_decode(np.uint8(0x08)) == 2.0 ** -6
    assert codecs.e4m3_decode(np.uint8(0x01)) == 2.0 ** -9
    assert codecs.e4m3_decode(np.uint8(0x38)) == 1.0
    assert codecs.e4m3_decode(np.uint8(0xC0)) == -2.0
    assert np.isnan(codecs.e4m3_decode(np.uint8(0x7F)))
    assert np.isnan(codecs.e4m3_decode(np.uint8(0xFF)))


def test_e4m3_matches_ml_dtypes_on_random_and_ties():
    _, vals = _finite_e4m3_values()
    pos = np.unique(vals[vals >= 0])
    mids = (pos[:-1] + pos[1:]) / 2          # every tie between neighbours
    x = np.concatenate([RNG.uniform(-448, 448, 20000), RNG.normal(0, 0.01, 20000),
                        mids, -mids, pos, -pos]).astype(np.float32)
    ours = codecs.e4m3_decode(codecs.e4m3_encode(x))
    ref = x.astype(ml_dtypes.float8_e4m3fn).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)
    tref = torch.from_numpy(x).to(torch.float8_e4m3fn).to(torch.float64).numpy()
    np.testing.assert_array_equal(ours, tref)


def test_e4m3_roundtrip_and_saturation():
    codes, vals = _finite_e4m3_values()
    back = codecs.e4m3_encode(vals.astype(np.float32))
    # -0 and +0 both finite; encoding keeps the sign bit
    np.testing.assert_array_equal(back, codes)
    assert codecs.e4m3_encode(np.float32(1000.0)) == 0x7E
    assert codecs.e4m3_encode(np.float32(-1e30)) == 0xFE
    assert codecs.e4m3_encode(np.float32(460.0)) == 0x7E


def test_e2m1_table_and_ml_dtypes():
    vals = codecs.e2m1_decode(np.arange(16, dtype=np.uint8))
    np.testing.assert_array_equal(vals[:8], [0, 0.5, 1, 1.5, 2, 3, 4, 6])
    np.testing.assert_array_equal(vals[8:], -np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6]))
    pos = np.array([0, 0.5, 1, 1.5, 2, 3, 4, 6])
    mids = (pos[:-1] + pos[1:]) / 2
    x = np.concatenate([RNG.uniform(-6, 6, 5000), mids, -mids, pos, -pos]).astype(np.float32)
    ours = codecs.e2m1_decode(codecs.e2m1_encode(x))
    ref = x.astype(ml_dtypes.float4_e2m1fn).astype(np.float64)
    np.testing.assert_array_equal(ours, ref)
    assert codecs.e2m1_decode(codecs.e2m1_encode(np.float32(7.9))) == 6.0
    # ties go to the even mantissa: 0.25 -> 0, 0.75 -> 1, 2.5 -> 2, 5 -> 4
    np.testing.assert_array_equal(codecs.e2m1_decode(codecs.e2m1_encode(
        np.array([0.25, 0.75, 2.5, 5.0], np.float32))), [0, 1, 2, 4])


def test_e2m1_packing_order():
    assert codecs.pack_e2m1(np.array([1, 2], np.uint8))[0] == 0x21
    c = RNG.integers(0, 16, (5, 32)).astype(np.uint8)
    np.testing.assert_array_equal(codecs.unpack_e2m1(codecs.pack_e2m1(c)), c)


def test_bf16_rounding_matches_libraries_and_avoids_double_rounding():
    x = np.concatenate([RNG.normal(0, 1, 20000), RNG.normal(0, 1e-30, 100),
                        RNG.uniform(-1e30, 1e30, 100)]).astype(np.float32)
    ours = codecs.round_to_bf16(x.astype(np.float64))
    np.testing.assert_array_equal(ours, x.astype(ml_dtypes.bfloat16).astype(np.float64))
    np.testing.assert_array_equal(ours, torch.from_numpy(x).bfloat16().double().numpy())
    # ties to even: 1 + 2^-8 -> 1 ; 1 + 3*2^-8 -> 1 + 2^-6
    assert codecs.round_to_bf16(np.array([1 + 2.0 ** -8]))[0] == 1.0
    assert codecs.round_to_bf16(np.array([1 + 3 * 2.0 ** -8]))[0] == 1 + 2.0 ** -6
    # a float64 just above a tie rounds up (a float32 detour would land on the tie and go down)
    assert codecs.round_to_bf16(np.array([1 + 2.0 ** -8 + 2.0 ** -40]))[0] == 1 + 2.0 ** -7
    bits = codecs.bf16_bits(np.array([1.0, -2.0]))
    np.testing.assert_array_equal(bits, [0x3F80, 0xC000])


def test_fp8_row_quantiser_bounds():
    x = RNG.normal(0, 1, (64, 128)).astype(np.float32)
    codes, scales = codecs.quant_fp8_rows(x)
    assert scales.dtype == np.float32
    np.testing.assert_array_equal(scales, (np.abs(x).max(1) / np.float32(448)).astype(np.float32))
    # the largest element of each row lands on +-448 (after float32 division it is within an ulp of 448)
    amax_pos = np.abs(x).argmax(1)
    top = codecs.e4m3_decode(codes[np.arange(64), amax_pos])
    np.testing.assert_array_equal(np.abs(top), 448.0)
    deq = codecs.dequant_fp8_rows(codes, scales)
    y = x / scales[:, None].astype(np.float64)
    err = np.abs(deq / scales[:, None] - y)
    bound = np.maximum(np.abs(y) * 2.0 ** -4, 2.0 ** -10) * (1 + 1e-6)
    assert np.all(err <= bound)
    zc, zs = codecs.quant_fp8_rows(np.zeros((2, 8), np.float32))
    assert np.all(zc == 0) and np.all(zs == 0)


def test_nvfp4_quantiser_exact_cases():
    # a block whose amax is 6 has scale exactly 1, so codes are the plain E2M1 codes
    x = np.array([6, -3, 0.5, 1.5, 2, -4, 1, 0.25] * 2, np.float32)[None]
    packed, sc = codecs.quant_nvfp4(x)
    assert codecs.e4m3_decode(sc)[0, 0] == 1.0
    np.testing.assert_array_equal(codecs.dequant_nvfp4(packed, sc)[0],
                                  [6, -3, 0.5, 1.5, 2, -4, 1, 0] * 2)
    # scaling a block by 2^k scales its scale by 2^k and keeps the codes
    p2, s2 = codecs.quant_nvfp4(x * np.float32(0.125))
    np.testing.assert_array_equal(p2, packed)
    assert codecs.e4m3_decode(s2)[0, 0] == 0.125
    r = RNG.normal(0, 1, (32, 128)).astype(np.float32)
    p, s = codecs.quant_nvfp4(r)
    assert p.shape == (32, 64) and s.shape == (32, 8)
    deq = codecs.dequant_nvfp4(p, s)
    sv = np.repeat(codecs.e4m3_decode(s), 16, axis=1)
    # error at most half of the widest E2M1 step (2, between 4 and 6) times the scale,
    # plus saturation when the rounded scale fell below amax/6 (at most 6/16 of a step)
    assert np.all(np.abs(deq - r) <= sv * 1.0 + 1e-6)


# ---------------------------------------------------------------------------
# compressor
# ---------------------------------------------------------------------------

def _rand_branch(n, c, m, rng=RNG):
    return dict(C_a=rng.normal(size=(n, c)), Z_a=rng.normal(size=(n, c)),
                B_a=rng.normal(0, 0.5, (m, c)), C_b=rng.normal(size=(n, c)),
                Z_b=rng.normal(size=(n, c)), B_b=rng.normal(0, 0.5, (m, c)))


def test_compressor_weights_sum_to_one_and_block0_padding():
    br = _rand_branch(64, 16, 4)
    for i in (0, 1, 7, 15):
        wgt = csa.compress_weights(br["Z_a"], br["B_a"], br["Z_b"], br["B_b"], 4, True, i)
        assert wgt.shape == (8, 16)
        np.testing.assert_allclose(wgt.sum(0), 1.0, rtol=0, atol=1e-12)
        if i == 0:
            assert np.all(wgt[:4] == 0.0)
        else:
            assert np.all(wgt[:4] > 0.0)
    br = _rand_branch(64, 16, 16)
    wgt = csa.compress_weights(br["Z_a"], br["B_a"], None, None, 16, False, 2)
    assert wgt.shape == (16, 16)
    np.testing.assert_allclose(wgt.sum(0), 1.0, atol=1e-12)


def test_compressor_m1_without_overlap_is_identity():
    br = _rand_branch(20, 8, 1)
    out = csa.compress_entries(br["C_a"], br["Z_a"], br["B_a"], None, None, None, 1, False,
                               np.arange(20), d_rope=0, theta=1e4, eps=1e-6, apply_norm=False)
    np.testing.assert_array_equal(out, br["C_a"])


def test_compressor_closed_form_two_rows_per_block():
    # m = 2, c = 1, entry 1 uses b-rows 0,1 (previous block) and a-rows 2,3 (current block).
    # Rows the entry must NOT read carry large logits / contents so any wrong pick shows.
    n, junk, junk_z = 6, 1000.0, 50.0
    C_a = np.full((n, 1), junk); C_b = np.full((n, 1), junk)
    Z_a = np.full((n, 1), junk_z); Z_b = np.full((n, 1), junk_z)
    Z_b[0:2, 0] = [0.0, 0.0]; C_b[0:2, 0] = [8.0, 0.0]
    Z_a[2:4, 0] = [math.log(2), math.log(2)]; C_a[2:4, 0] = [0.0, 4.0]
    B_b = np.array([[0.0], [math.log(3)]])   # bias by row position inside the block
    B_a = np.zeros((2, 1))
    out = csa.compress_pool(C_a, Z_a, B_a, C_b, Z_b, B_b, 2, True, [1])
    # weights e^[0, ln3, ln2, ln2] / 8 = [1, 3, 2, 2] / 8 -> (8*1 + 0*3 + 0*2 + 4*2) / 8 = 2
    np.testing.assert_allclose(out[0, 0], 2.0, rtol=1e-14)
    wgt = csa.compress_weights(Z_a, B_a, Z_b, B_b, 2, True, 1)
    np.testing.assert_allclose(wgt[:, 0], [1 / 8, 3 / 8, 2 / 8, 2 / 8], rtol=1e-14)


def test_compressor_constant_content_is_preserved():
    br = _rand_branch(32, 8, 4)
    v = RNG.normal(size=8)
    br["C_a"][:] = v
    br["C_b"][:] = v
    out = csa.compress_pool(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"], 4,
                            True, np.arange(1, 8))
    np.testing.assert_allclose(out, np.broadcast_to(v, out.shape), rtol=1e-13)


def test_compressor_receptive_field_is_8_rows_at_stride_4():
    """Perturbing raw row r changes entry r//4 (through C_a) or entry r//4 + 1 (through C_b) only."""
    n, c, m = 64, 4, 4
    br = _rand_branch(n, c, m)
    E = n // m
    base = csa.compress_pool_vec(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"],
                                 m, True, 0, E)
    for name, expect in (("C_a", lambda r: {r // m}), ("Z_a", lambda r: {r // m}),
                         ("C_b", lambda r: {r // m + 1} - {E}), ("Z_b", lambda r: {r // m + 1} - {E})):
        for r in (0, 3, 17, 62, 63):
            pert = {k2: v.copy() for k2, v in br.items()}
            pert[name][r] += 1.0
            out = csa.compress_pool_vec(pert["C_a"], pert["Z_a"], pert["B_a"], pert["C_b"],
                                        pert["Z_b"], pert["B_b"], m, True, 0, E)
            changed = set(np.nonzero(np.any(out != base, axis=1))[0].tolist())
            assert changed == expect(r), (name, r, changed)


def test_compress_pool_vec_equals_per_entry_loop():
    for overlap, m in ((True, 4), (False, 8), (True, 1)):
        br = _rand_branch(96, 12, m)
        E = 96 // m
        a = csa.compress_pool(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"], m,
                              overlap, np.arange(E))
        for i0, cnt in ((0, E), (3, E - 3), (0, 1), (E - 1, 1)):
            b = csa.compress_pool_vec(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"],
                                      br["B_b"], m, overlap, i0, cnt)
            np.testing.assert_allclose(b, a[i0:i0 + cnt], rtol=1e-13, atol=1e-15)
        r = csa.compress_range(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"], m,
                               overlap, 0, E, 4, 1e4, 1e-6, chunk_rows=7)
        e = csa.compress_entries(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"],
                                 m, overlap, np.arange(E), 4, 1e4, 1e-6)
        np.testing.assert_allclose(r, e, rtol=1e-13, atol=1e-15)


def test_rmsnorm_unit_rms_and_scale_invariance():
    x = RNG.normal(size=(10, 64)) * 3.0
    y = csa.rms_norm(x, 0.0)
    np.testing.assert_allclose(np.sqrt(np.mean(y * y, 1)), 1.0, rtol=1e-14)
    np.testing.assert_allclose(csa.rms_norm(7.5 * x, 0.0), y, rtol=1e-13)
    # eps enters inside the root: a zero vector stays zero, a tiny vector is damped
    assert np.all(csa.rms_norm(np.zeros((1, 4)), 1e-6) == 0)
    np.testing.assert_allclose(csa.rms_norm(np.full((1, 4), 1e-3), 1e-6)[0, 0],
                               1e-3 / math.sqrt(1e-6 + 1e-6), rtol=1e-14)


def test_rope_closed_forms():
    c, d_r, th = 24, 16, 10000.0
    # pair j = 1 rotates at theta^(-2/16) = 10^(-1/2)
    x = np.zeros((1, c)); x[0, c - d_r + 2] = 1.0
    y = csa.rope_partial(x, [1], d_r, th)
    f1 = 10.0 ** -0.5
    np.testing.assert_allclose(y[0, c - d_r + 2:c - d_r + 4], [math.cos(f1), math.sin(f1)], rtol=1e-15)
    # pair 0 has frequency 1; the second element of a pair rotates to (-sin, cos)
    x = np.zeros((1, c)); x[0, c - d_r + 1] = 1.0
    y = csa.rope_partial(x, [3], d_r, th)
    np.testing.assert_allclose(y[0, c - d_r:c - d_r + 2], [-math.sin(3), math.cos(3)], rtol=1e-15)
    # the leading c - d_r dims never move; norms of pairs are kept; p = 0 is the identity
    x = RNG.normal(size=(5, c))
    y = csa.rope_partial(x, [0, 5, 77, 4096, 1 << 20], d_r, th)
    np.testing.assert_array_equal(y[:, :c - d_r], x[:, :c - d_r])
    np.testing.assert_array_equal(y[0], x[0])
    pn = lambda z: np.hypot(z[:, c - d_r::2], z[:, c - d_r + 1::2])
    np.testing.assert_allclose(pn(y), pn(x), rtol=1e-13)
    # rotations compose additively in the position
    a = csa.rope_partial(csa.rope_partial(x, [3] * 5, d_r, th), [11] * 5, d_r, th)
    np.testing.assert_allclose(a, csa.rope_partial(x, [14] * 5, d_r, th), atol=1e-12)


def test_compressed_entry_anchor_and_norm_closed_form():
    """A constant one-hot content gives entry i = sqrt(c) * (cos(m i), sin(m i)) on rotary pair 0."""
    n, c, m, d_r = 64, 8, 4, 4
    br = _rand_branch(n, c, m)
    v = np.zeros(c); v[c - d_r] = 2.5
    br["C_a"][:] = v; br["C_b"][:] = v
    out = csa.compress_entries(br["C_a"], br["Z_a"], br["B_a"], br["C_b"], br["Z_b"], br["B_b"], m,
                               True, np.arange(n // m), d_r, 1e4, 0.0)
    i = np.arange(n // m)
    np.testing.assert_allclose(out[:, c - d_r], math.sqrt(c) * np.cos(m * i), atol=1e-12)
    np.testing.assert_allclose(out[:, c - d_r + 1], math.sqrt(c) * np.sin(m * i), atol=1e-12)
    np.testing.assert_allclose(out[:, :c - d_r], 0.0, atol=1e-12)


# ---------------------------------------------------------------------------
# indexer
# ---------------------------------------------------------------------------

def test_indexer_closed_form_one_hot():
    d = 8
    q = np.zeros((1, 2, d)); q[0, 0, 3] = 2.0; q[0, 1, 3] = -1.0
    k = np.zeros((2, d)); k[0, 3] = 3.0; k[1, 3] = -2.0
    w = np.array([[0.5, 0.25]])
    sc = csa.index_scores(q, w, k, np.array([7]), m=4, out_dtype="f64")
    # s=0: 0.5*relu(6) + 0.25*relu(-3) = 3 ; s=1: 0.5*relu(-4) + 0.25*relu(2) = 0.5
    np.testing.assert_array_equal(sc[0], [3.0, 0.5])


def test_indexer_single_head_is_relu_dot():
    q = RNG.normal(size=(3, 1, 16)); k = RNG.normal(size=(40, 16))
    sc = csa.index_scores(q, np.ones((3, 1)), k, np.array([1000] * 3), m=4, out_dtype="f64")
    ref = np.maximum(q[:, 0, :] @ k.T, 0.0)
    np.testing.assert_allclose(sc, ref, rtol=1e-14)


def test_indexer_causal_mask_and_rounding():
    q = RNG.normal(size=(6, 2, 4)); k = RNG.normal(size=(4, 4)); w = np.ones((6, 2))
    t = np.array([0, 2, 3, 4, 7, 15])
    sc = csa.index_scores(q, w, k, t, m=4, out_dtype="bf16")
    vis = [0, 0, 1, 1, 2, 4]    # E(t) = floor((t+1)/4): block s ends at 4s+3 <= t
    for r in range(6):
        assert np.all(np.isinf(sc[r, vis[r]:]) & (sc[r, vis[r]:] < 0))
        assert np.all(np.isfinite(sc[r, :vis[r]]))
    fin = sc[np.isfinite(sc)]
    np.testing.assert_array_equal(fin, codecs.round_to_bf16(fin))


# ---------------------------------------------------------------------------
# top-k
# ---------------------------------------------------------------------------

def test_topk_equals_brute_force_sort_with_ties():
    for trial in range(40):
        E = int(RNG.integers(1, 40))
        k = int(RNG.integers(1, 20))
        T = 5
        sc = RNG.integers(-3, 4, size=(T, E)).astype(np.float64)   # many exact ties
        m = int(RNG.integers(1, 5))
        t = RNG.integers(0, m * E + 3, size=T)
        idx, cnt = csa.topk(sc, t, m, k)
        for r in range(T):
            ev = min((int(t[r]) + 1) // m, E)
            cand = sorted(range(ev), key=lambda s: (-sc[r, s], s))[:k]
            want = sorted(cand)
            assert cnt[r] == len(want)
            assert list(idx[r, :cnt[r]]) == want
            assert np.all(idx[r, cnt[r]:] == -1)
            if cnt[r]:
                assert idx[r, cnt[r] - 1] < ev          # causality


# ---------------------------------------------------------------------------
# attention
# ---------------------------------------------------------------------------

def test_attention_equals_softmax_with_sink_column():
    H, d, R = 4, 16, 9
    q = RNG.normal(size=(H, d)); rows = RNG.normal(size=(R, d)); sink = RNG.normal(size=H)
    o, lse = csa.attend(q, rows, sink, 0.25)
    logits = np.concatenate([0.25 * q @ rows.T, sink[:, None]], axis=1)
    p = scipy.special.softmax(logits, axis=1)
    vals = np.concatenate([rows, np.zeros((1, d))], axis=0)
    np.testing.assert_allclose(o, p @ vals, rtol=1e-12, atol=1e-14)
    np.testing.assert_allclose(lse, scipy.special.logsumexp(logits, axis=1), rtol=1e-13)
    o2, _ = csa.attend(q, rows, np.full(H, -np.inf), 0.25)
    np.testing.assert_allclose(o2, scipy.special.softmax(0.25 * q @ rows.T, axis=1) @ rows,
                               rtol=1e-12, atol=1e-14)


def test_attention_single_row_closed_form_and_stability():
    q = np.array([[1.0, 2.0]]); row = np.array([[0.5, -1.0]]); sink = np.array([0.3])
    o, _ = csa.attend(q, row, sink, 2.0)
    l = 2.0 * (0.5 - 2.0)
    np.testing.assert_allclose(o[0], row[0] * math.exp(l) / (math.exp(l) + math.exp(0.3)), rtol=1e-14)
    big = csa.attend(q * 1e4, np.array([[1.0, 1.0], [2.0, 2.0]]), sink, 1.0)[0]
    assert np.all(np.isfinite(big))
    np.testing.assert_allclose(big[0], [2.0, 2.0])


def test_window_rows_and_topk_all_equals_dense():
    assert list(csa.window_rows(0, 16)) == [0]
    assert list(csa.window_rows(5, 3)) == [3, 4, 5]
    n, m, H, d, n_w = 64, 4, 2, 8, 5
    kv = RNG.normal(size=(n // m, d)); win = RNG.normal(size=(n, d))
    q = RNG.normal(size=(n, H, d)); sink = RNG.normal(size=H)
    t = np.arange(n)
    sc = RNG.normal(size=(n, n // m))
    idx, cnt = csa.topk(sc, t, m, n // m)          # k >= E(t): every visible entry
    o1, l1 = csa.sparse_attn(q, kv, idx, cnt, win, t, sink, n_w, 0.3)
    o2, l2 = csa.dense_attn(q, kv, win, t, sink, n_w, 0.3, m)
    np.testing.assert_allclose(o1, o2, rtol=1e-13, atol=1e-15)
    # query t with no visible entry attends to its window and the sink only
    o0, _ = csa.attend(q[2], win[0:3], sink, 0.3)
    np.testing.assert_allclose(o1[2], o0, rtol=1e-14)


# ---------------------------------------------------------------------------
# geometry printed on the pages
# ---------------------------------------------------------------------------

def test_geometry_golden():
    g = json.load(open(os.path.join(GOLDEN, "geometry.json")))
    n = g["context_1m_tokens"]["value"]
    m4, m128 = g["c4a_stride"]["value"], g["c128a_stride"]["value"]
    br = _rand_branch(16, 2, m4)
    assert csa.compress_weights(br["Z_a"], br["B_a"], br["Z_b"], br["B_b"], m4, True, 2).shape[0] \
        == g["c4a_rows_per_entry"]["value"]
    assert csa.visible_entries(n - 1, m4) == n // m4
    assert abs(n // m4 - g["c4a_entries_at_1m_approx"]["value"]) <= \
        g["c4a_entries_at_1m_approx"]["rel_tol"] * g["c4a_entries_at_1m_approx"]["value"]
    assert csa.visible_entries(n - 1, m128) == g["c128a_entries_at_1m_max"]["value"]
    # cache accounting: 320 MiB / 262144 entries = 1280 B = bf16 latent (512) + bf16 index key (128)
    per_entry = g["csa_layer_cache_mib_at_1m"]["value"] * 2 ** 20 / (n // m4)
    assert per_entry == 2 * (g["latent_dim"]["value"] + g["index_key_dim"]["value"])
    assert g["hca_layer_cache_mib_at_1m"]["value"] * 2 ** 20 / (n // m128) == 2 * g["latent_dim"]["value"]
    v32 = g["v32_bytes_per_token_layer"]["value"] * n * g["v32_total_gib"]["layers"] / 2 ** 30
    assert abs(v32 - g["v32_total_gib"]["value"]) <= g["v32_total_gib"]["abs_tol"]


# ---------------------------------------------------------------------------
# compositions
# ---------------------------------------------------------------------------

def test_prefill_pipeline_tiny_consistency():
    """The prefill composition agrees with its stages and with the decode composition."""
    n, m, c, cI, H, HI = 64, 4, 16, 8, 2, 2
    rng = np.random.default_rng(7)
    main = _rand_branch(n, c, m, rng)
    index = _rand_branch(n, cI, m, rng)
    q = rng.normal(size=(n, H, c)); qI = rng.normal(size=(n, HI, cI))
    w = rng.uniform(size=(n, HI)) / 4; sink = rng.normal(size=H)
    kw = dict(m=m, d_rope=4, theta=1e4, eps=1e-6, n_w=4, scale=0.25, kv_dtype="f32")
    pre = pipeline.csa_prefill(main, index, q, qI, w, sink, k=3, idx_dtype="fp8",
                               score_dtype="bf16", **kw)
    assert pre["idx"].shape == (n, 3)
    t = n - 1
    dec = pipeline.csa_decode_seq(main, index, q[t], qI[t], w[t], sink, L=n, k=3, idx_dtype="fp8", **kw)
    np.testing.assert_array_equal(dec["idx"], pre["idx"][t])
    np.testing.assert_allclose(dec["out_f64"], pre["out_f64"][t], rtol=1e-12)
    np.testing.assert_allclose(dec["new_entry"], pre["kv"][n // m - 1], rtol=1e-13)
