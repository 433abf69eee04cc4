"""Stage-isolated parity of the CUDA kernels against the CPU oracle.

Every stage gets identical inputs on both sides (drawn by the seeded
generator, or produced by the oracle for the stage's own inputs), and every
call goes through the C ABI.  Sizes span several tiles and a ragged tail.
"""

import math

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import synth
from oracle import codecs, csa

from helpers import (assert_abs_close, assert_rel_close, f64, nvfp4_scales_from_tiled,
                     nvfp4_scales_to_tiled, topk_band_check)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _branch(b, n, c, m, seed, dtype, overlap=True, device=DEV):
    d = {}
    d["C_a"] = synth.draw("C_a", (b, n, c), seed, device, dtype)
    d["Z_a"] = synth.draw("Z_a", (b, n, c), seed, device, dtype)
    d["B_a"] = synth.draw("B_a", (m, c), seed, device, "f32", spread=0.5)
    if overlap:
        d["C_b"] = synth.draw("C_b", (b, n, c), seed, device, dtype)
        d["Z_b"] = synth.draw("Z_b", (b, n, c), seed, device, dtype)
        d["B_b"] = synth.draw("B_b", (m, c), seed, device, "f32", spread=0.5)
    return d


def _oracle_compress(d, s, m, overlap, E, d_rope, apply_norm=True, eps=1e-6):
    g = {k: f64(v[s]) if v.dim() == 3 else f64(v) for k, v in d.items()}
    return csa.compress_range(g["C_a"], g["Z_a"], g["B_a"], g.get("C_b"), g.get("Z_b"), g.get("B_b"),
                              m, overlap, 0, E, d_rope, 1e4, eps, apply_norm)


def _run_compress(d, b, n, c, m, overlap, E, d_rope, in_dt, out_dt, apply_norm=True, E_cap=None,
                  entry_begin=0):
    E_cap = E_cap or E
    if out_dt in ("f32", "bf16"):
        out = torch.zeros((b, E_cap, c), dtype=torch.float32 if out_dt == "f32" else torch.bfloat16,
                          device=DEV)
        sc = None
    elif out_dt == "fp8":
        out = torch.zeros((b, E_cap, c), dtype=torch.uint8, device=DEV)
        sc = torch.zeros((b, E_cap), dtype=torch.float32, device=DEV)
    else:
        out = torch.zeros((b, E_cap, c // 2), dtype=torch.uint8, device=DEV)
        sc = torch.zeros((b, (E_cap + 127) // 128 * 128, c // 16), dtype=torch.uint8, device=DEV)
    p = L.CompressParams(m=m, overlap=int(overlap), c=c, d_rope=d_rope, rope_theta=1e4, eps=1e-6,
                         apply_norm=int(apply_norm), in_dtype=L.DTYPE[in_dt],
                         out_dtype=L.DTYPE[out_dt])
    L.csa_compress(p, d["C_a"], d["Z_a"], d["B_a"], d.get("C_b"), d.get("Z_b"), d.get("B_b"), b, n,
                   entry_begin, E - entry_begin, E_cap, out, sc)
    torch.cuda.synchronize()
    return out, sc


@pytest.mark.parametrize("c,d_rope,seed", [(64, 16, 0), (32, 16, 1)])
def test_compress_f32_tiny(c, d_rope, seed):
    b, n, m = 1, 1024, 4
    d = _branch(b, n, c, m, seed, "f32")
    out, _ = _run_compress(d, b, n, c, m, True, n // m, d_rope, "f32", "f32")
    ref = _oracle_compress(d, 0, m, True, n // m, d_rope)
    assert_rel_close(f64(out[0]), ref, 1e-5, "compress f32")


def test_compress_bf16_c4a_ragged_and_partial():
    b, n, c, m = 2, 520, 512, 4          # 130 entries: not a multiple of any tile
    E = n // m
    d = _branch(b, n, c, m, 11, "bf16")
    out32, _ = _run_compress(d, b, n, c, m, True, E, 64, "bf16", "f32")
    out16, _ = _run_compress(d, b, n, c, m, True, E, 64, "bf16", "bf16")
    for s in range(b):
        ref = _oracle_compress(d, s, m, True, E, 64)
        assert_rel_close(f64(out32[s]), ref, 1e-5, "compress bf16->f32")
        assert_rel_close(f64(out16[s]), ref, 2e-2, "compress bf16->bf16")
        # bf16 output is the round-to-nearest of the float32 result (torch's own cast)
        assert torch.equal(out16[s], out32[s].to(torch.bfloat16))
    # updating a tail range leaves the rest of the cache untouched
    part, _ = _run_compress(d, b, n, c, m, True, E, 64, "bf16", "f32", E_cap=E + 3, entry_begin=100)
    assert torch.all(part[:, :100] == 0) and torch.all(part[:, E:] == 0)
    assert torch.equal(part[:, 100:E], out32[:, 100:E])


def test_compress_hca_c128a():
    b, n, c, m = 2, 128 * 5, 512, 128
    d = _branch(b, n, c, m, 12, "bf16", overlap=False)
    out, _ = _run_compress(d, b, n, c, m, False, n // m, 64, "bf16", "f32")
    for s in range(b):
        assert_rel_close(f64(out[s]), _oracle_compress(d, s, m, False, n // m, 64), 1e-5, "c128a")


def test_compress_m1_is_identity():
    b, n, c = 2, 40, 64
    d = _branch(b, n, c, 1, 13, "f32", overlap=False)
    out, _ = _run_compress(d, b, n, c, 1, False, n, 0, "f32", "f32", apply_norm=False)
    assert torch.equal(out, d["C_a"])


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
def test_compress_index_branch_quantised(fmt):
    b, n, c, m = 2, 1000, 128, 4
    E = n // m
    d = _branch(b, n, c, m, 14, "bf16")
    codes, sc = _run_compress(d, b, n, c, m, True, E, 64, "bf16", fmt)
    out32, _ = _run_compress(d, b, n, c, m, True, E, 64, "bf16", "f32")
    # the fused quantiser equals the stand-alone quantiser applied to the kernel's own float32 rows
    rows = b * E
    c2 = torch.empty_like(codes)
    s2 = torch.empty((rows,), dtype=torch.float32, device=DEV) if fmt == "fp8" else \
        torch.empty((rows, c // 16), dtype=torch.uint8, device=DEV)
    L.csa_quantize(L.CSA_F32, L.DTYPE[fmt], out32, rows, c, c2, s2)
    torch.cuda.synchronize()
    if fmt == "nvfp4":   # the cache keeps its scales in the tiled layout; the quantiser row-major
        sc = torch.from_numpy(nvfp4_scales_from_tiled(sc.cpu().numpy(), E)).to(DEV)
    assert torch.equal(c2, codes) and torch.equal(s2.reshape(sc.shape), sc)
    for s in range(b):
        ref = _oracle_compress(d, s, m, True, E, 64)
        assert_rel_close(f64(out32[s]), ref, 1e-5, "index branch f32")
        # Against the oracle's own entries.  The kernel's float32 rows are within
        # 1e-5 * (|x| + rms) of the oracle's (checked above), so a scale or a code may
        # differ only where the oracle's value lies that close to the rounding
        # boundary between the two: the midpoint of the two neighbouring grid values.
        rms = np.sqrt(np.mean(ref ** 2, axis=1, keepdims=True))
        tol = 2e-5 * (np.abs(ref) + rms)
        gc, gs = codes[s].cpu().numpy(), sc[s].cpu().numpy()
        if fmt == "fp8":
            rc, rs = codecs.quant_fp8_rows(ref.astype(np.float32))
            np.testing.assert_allclose(gs, rs, rtol=1e-5)
            gv, rv = codecs.e4m3_decode(gc), codecs.e4m3_decode(rc)
            x_over_s = ref / rs[:, None]
            bound = tol / rs[:, None]
        else:
            rc, rs = codecs.quant_nvfp4(ref.astype(np.float32))
            # a block scale differs only where amax / 6 straddles an E4M3 boundary
            gsv, rsv = codecs.e4m3_decode(gs), codecs.e4m3_decode(rs)
            amax6 = np.abs(ref).reshape(E, -1, 16).max(axis=2) / 6.0
            bad = gs != rs
            assert np.all(np.abs(amax6[bad] - 0.5 * (gsv[bad] + rsv[bad])) <=
                          2e-5 * amax6[bad]), "scale differs away from a rounding boundary"
            same_blk = np.repeat(~bad, 16, axis=1)
            gv = np.where(same_blk, codecs.e2m1_decode(codecs.unpack_e2m1(gc)), 0.0)
            rv = np.where(same_blk, codecs.e2m1_decode(codecs.unpack_e2m1(rc)), 0.0)
            sv = np.repeat(rsv, 16, axis=1)
            x_over_s = ref / np.where(sv > 0, sv, 1.0)
            bound = tol / np.where(sv > 0, sv, 1.0)
        diff = gv != rv
        assert np.all(np.abs(x_over_s[diff] - 0.5 * (gv[diff] + rv[diff])) <= bound[diff]), \
            "a code differs away from a rounding boundary"


@pytest.mark.parametrize("fmt", ["fp8", "nvfp4"])
@pytest.mark.parametrize("in_dt", ["bf16", "f32"])
def test_quantize_bit_exact(fmt, in_dt):
    rows, d = 777, 128
    x = synth.draw("q_I", (rows, d), 21, DEV, in_dt)
    x[5] = 0
    x[6] *= 1e-3
    x[7] *= 300
    cbytes = d if fmt == "fp8" else d // 2
    codes = torch.empty((rows, cbytes), dtype=torch.uint8, device=DEV)
    sc = torch.empty((rows,), dtype=torch.float32, device=DEV) if fmt == "fp8" else \
        torch.empty((rows, d // 16), dtype=torch.uint8, device=DEV)
    L.csa_quantize(L.DTYPE[in_dt], L.DTYPE[fmt], x, rows, d, codes, sc)
    torch.cuda.synchronize()
    xs = x.float().cpu().numpy()
    c_ref, s_ref = codecs.quant_fp8_rows(xs) if fmt == "fp8" else codecs.quant_nvfp4(xs)
    np.testing.assert_array_equal(codes.cpu().numpy(), c_ref)
    np.testing.assert_array_equal(sc.cpu().numpy(), s_ref)


def _index_inputs(b, T, E, H, d, fmt, seed):
    """Quantised q/k produced by the oracle's quantiser, so both sides score identical codes."""
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(b, T, H, d)).astype(np.float32)
    k = rng.normal(size=(b, E, d)).astype(np.float32)
    w = (rng.uniform(size=(b, T, H)) / 64).astype(np.float32)
    if fmt == "f32":
        return dict(q=q, qs=None, k=k, ks=None, w=w, qd=q.astype(np.float64), kd=k.astype(np.float64))
    if fmt == "fp8":
        qc, qs = codecs.quant_fp8_rows(q)
        kc, ks = codecs.quant_fp8_rows(k)
        return dict(q=qc, qs=qs, k=kc, ks=ks, w=w, qd=codecs.dequant_fp8_rows(qc, qs),
                    kd=codecs.dequant_fp8_rows(kc, ks))
    qc, qs = codecs.quant_nvfp4(q)
    kc, ks = codecs.quant_nvfp4(k)
    # the library reads key scales in its tiled layout (query scales stay row-major)
    return dict(q=qc, qs=qs, k=kc, ks=nvfp4_scales_to_tiled(ks), w=w,
                qd=codecs.dequant_nvfp4(qc, qs), kd=codecs.dequant_nvfp4(kc, ks))


def _dev(a):
    return None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to(DEV)


@pytest.mark.parametrize("fmt,H,d,T,E,m,score", [
    ("fp8", 64, 128, 1, 1000, 4, "bf16"),     # decode-like, ragged 128-entry tiles
    ("nvfp4", 64, 128, 1, 1000, 4, "bf16"),
    ("fp8", 64, 128, 1, 40000, 4, "bf16"),    # long rows: CTAs that take two work units
    ("nvfp4", 64, 128, 1, 40000, 4, "bf16"),
    ("fp8", 64, 128, 37, 80, 4, "bf16"),      # prefill-like: causal mask across queries
    ("f32", 4, 32, 50, 64, 4, "f32"),         # tiny fp32 configuration
])
def test_index_scores(fmt, H, d, T, E, m, score):
    b = 2
    x = _index_inputs(b, T, E, H, d, fmt, 31)
    if T == 1:
        qpos = np.full((b, T), m * E - 1, dtype=np.int32)
        qpos[1, 0] = m * 600 + 2            # second sequence sees only 600 entries
    else:
        qpos = np.tile(np.arange(T, dtype=np.int32) * (m * E // T) + 3, (b, 1))
    scores = torch.empty((b, T, E), dtype=torch.bfloat16 if score == "bf16" else torch.float32,
                         device=DEV)
    p = L.IndexParams(H_I=H, d_I=d, m=m, qk_dtype=L.DTYPE[fmt], score_dtype=L.DTYPE[score])
    L.csa_index_scores(p, _dev(x["q"]), _dev(x["qs"]), _dev(x["w"]), _dev(x["k"]), _dev(x["ks"]),
                       _dev(qpos), b, T, E, E, scores)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0      # no bounded wait gave up
    g = f64(scores)
    for s in range(b):
        exact = csa.index_scores(x["qd"][s], x["w"][s], x["kd"][s], qpos[s], m, "f64")
        fin = np.isfinite(exact)
        np.testing.assert_array_equal(np.isfinite(g[s]), fin)
        assert np.all(np.isneginf(g[s][~fin]))
        # float32 accumulation then one rounding: within one bf16 ulp (or float32 rel 1e-5)
        tol = (bf16_ulp_arr(exact[fin]) * 1.01) if score == "bf16" else 1e-5 * (np.abs(exact[fin]) + 1e-3)
        err = np.abs(g[s][fin] - exact[fin])
        assert np.all(err <= tol + 1e-7), np.max(err - tol)


def bf16_ulp_arr(x):
    from helpers import bf16_ulp
    return bf16_ulp(x)


@pytest.mark.parametrize("score", ["bf16", "f32"])
def test_topk_bit_exact(score):
    b, T, E, m = 2, 6, 3000, 4
    rng = np.random.default_rng(41)
    sc = np.round(rng.normal(size=(b, T, E)) * 8) / 8           # heavy ties
    sc[:, 1] = rng.normal(size=E)
    sc[:, 2] = 0.0                                               # all tied
    qpos = np.array([[m * E - 1, m * E - 1, m * E - 1, 4 * 300 + 1, 9, 0]] * b, dtype=np.int32)
    qpos[1, 4] = 4 * 517 - 1                                     # E(t) = 517 > k
    for k in (16, 512):
        tdt = torch.bfloat16 if score == "bf16" else torch.float32
        st = torch.from_numpy(sc).to(tdt).to(DEV)
        idx = torch.empty((b, T, k), dtype=torch.int32, device=DEV)
        cnt = torch.empty((b, T), dtype=torch.int32, device=DEV)
        L.csa_topk(st, L.DTYPE[score], _dev(qpos), m, b, T, E, k, idx, cnt)
        torch.cuda.synchronize()
        stored = f64(st)
        for s in range(b):
            ri, rc = csa.topk(stored[s], qpos[s], m, k)
            np.testing.assert_array_equal(cnt[s].cpu().numpy(), rc)
            np.testing.assert_array_equal(idx[s].cpu().numpy(), ri)


def test_topk_1m_row():
    E, k, m = 262144, 1024, 4
    sc = synth.draw("q", (1, 1, E), 42, "cpu", "bf16")
    st = sc.to(DEV)
    qpos = torch.full((1, 1), m * E - 1, dtype=torch.int32, device=DEV)
    idx = torch.empty((1, 1, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((1, 1), dtype=torch.int32, device=DEV)
    wsb = L.csa_topk_workspace_size(L.CSA_BF16, 1, 1, E, k)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_topk(st, L.CSA_BF16, qpos, m, 1, 1, E, k, idx, cnt, ws, wsb)
    torch.cuda.synchronize()
    ri, rc = csa.topk(f64(sc)[0], np.array([m * E - 1]), m, k)
    np.testing.assert_array_equal(idx[0].cpu().numpy(), ri)


@pytest.mark.parametrize("E,k,ties", [(40000, 1024, False), (40000, 1024, True), (70000, 16, True)])
def test_topk_chunked_rows_bit_exact(E, k, ties):
    """Rows longer than one CTA: per-chunk top-k then top-k of the candidates; ties across
    chunk borders must still go to the lowest entries."""
    b, T, m = 2, 3, 4
    rng = np.random.default_rng(E + k)
    sc = rng.normal(size=(b, T, E))
    if ties:
        sc = np.round(sc * 2) / 2
    qpos = np.array([[m * E - 1, m * 20000 + 1, m * 700 - 1]] * b, dtype=np.int32)
    st = torch.from_numpy(sc).to(torch.bfloat16).to(DEV)
    idx = torch.empty((b, T, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((b, T), dtype=torch.int32, device=DEV)
    wsb = L.csa_topk_workspace_size(L.CSA_BF16, b, T, E, k)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_topk(st, L.CSA_BF16, _dev(qpos), m, b, T, E, k, idx, cnt, ws, wsb)
    torch.cuda.synchronize()
    stored = f64(st)
    for s_ in range(b):
        ri, rc = csa.topk(stored[s_], qpos[s_], m, k)
        np.testing.assert_array_equal(cnt[s_].cpu().numpy(), rc)
        np.testing.assert_array_equal(idx[s_].cpu().numpy(), ri)


@pytest.mark.parametrize("E,k,rows", [(40000, 20000, 3), (1 << 20, 1024, 1)])
def test_topk_radix_path_bit_exact(E, k, rows):
    """Shapes no search plan covers (k above 16384; a row beyond a 16-CTA cluster whose
    per-chunk candidates overflow one CTA) take the radix select; it is exact too."""
    m = 4
    rng = np.random.default_rng(E + k)
    sc = rng.normal(size=(rows, 1, E))
    sc[0, 0, ::3] = np.round(sc[0, 0, ::3] * 2) / 2                # ties
    qpos = np.full((rows, 1), m * E - 1, dtype=np.int32)
    if rows > 2:
        qpos[2, 0] = m * (k + 3) - 1                               # E(t) = k + 3
    assert L.csa_topk_workspace_size(L.CSA_BF16, rows, 1, E, k) == 0
    st = torch.from_numpy(sc).to(torch.bfloat16).to(DEV)
    idx = torch.empty((rows, 1, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((rows, 1), dtype=torch.int32, device=DEV)
    L.csa_topk(st, L.CSA_BF16, _dev(qpos), m, rows, 1, E, k, idx, cnt)
    torch.cuda.synchronize()
    stored = f64(st)
    for r in range(rows):
        ri, rc = csa.topk(stored[r], qpos[r], m, k)
        np.testing.assert_array_equal(cnt[r].cpu().numpy(), rc)
        np.testing.assert_array_equal(idx[r].cpu().numpy(), ri)


@pytest.mark.parametrize("score", ["bf16", "f32"])
@pytest.mark.parametrize("E,k,b", [(16384, 512, 16), (262144, 1024, 4), (9000, 512, 3)])
def test_topk_cluster_rows_bit_exact(score, E, k, b):
    """Few long rows, each spread over a cluster of CTAs: ties across the CTAs' slice
    borders go to the lowest entries, and short visible prefixes leave whole CTAs empty."""
    m = 4
    rng = np.random.default_rng(E + k + b)
    sc = rng.normal(size=(b, 1, E))
    sc[1::2] = np.round(sc[1::2] * 2) / 2                       # heavy ties on odd rows
    sc[-1, 0, : E // 2] = 0.0                                    # a tied plateau
    qpos = np.full((b, 1), m * E - 1, dtype=np.int32)
    qpos[1, 0] = m * (k + 5) - 1                                 # E(t) = k + 5
    qpos[2 % b, 0] = m * (E // 3) + 2                            # ragged prefix
    if b > 3:
        qpos[3, 0] = m * (k - 7)                                 # E(t) < k: all kept
    tdt = torch.bfloat16 if score == "bf16" else torch.float32
    st = torch.from_numpy(sc).to(tdt).to(DEV)
    idx = torch.empty((b, 1, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((b, 1), dtype=torch.int32, device=DEV)
    wsb = L.csa_topk_workspace_size(L.DTYPE[score], b, 1, E, k)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_topk(st, L.DTYPE[score], _dev(qpos), m, b, 1, E, k, idx, cnt, ws, wsb)
    torch.cuda.synchronize()
    stored = f64(st)
    for s_ in range(b):
        ri, rc = csa.topk(stored[s_], qpos[s_], m, k)
        np.testing.assert_array_equal(cnt[s_].cpu().numpy(), rc)
        np.testing.assert_array_equal(idx[s_].cpu().numpy(), ri)


def test_topk_rows_beyond_a_cluster():
    """Rows longer than 16 x 16384 entries take the chunk pass + candidate pass."""
    E, k, m, b = 300000, 512, 4, 2
    rng = np.random.default_rng(7)
    sc = np.round(rng.normal(size=(b, 1, E)) * 4) / 4
    qpos = np.array([[m * E - 1], [m * 280001 + 3]], dtype=np.int32)
    st = torch.from_numpy(sc).to(torch.bfloat16).to(DEV)
    idx = torch.empty((b, 1, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((b, 1), dtype=torch.int32, device=DEV)
    wsb = L.csa_topk_workspace_size(L.CSA_BF16, b, 1, E, k)
    assert wsb > 0
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_topk(st, L.CSA_BF16, _dev(qpos), m, b, 1, E, k, idx, cnt, ws, wsb)
    torch.cuda.synchronize()
    stored = f64(st)
    for s_ in range(b):
        ri, rc = csa.topk(stored[s_], qpos[s_], m, k)
        np.testing.assert_array_equal(cnt[s_].cpu().numpy(), rc)
        np.testing.assert_array_equal(idx[s_].cpu().numpy(), ri)


def _attn_case(b, T, H, d, E, n, k, n_w, dtype, dense, seed):
    rng = np.random.default_rng(seed)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    q = synth.draw("q", (b, T, H, d), seed, DEV, dtype)
    kv = synth.draw("C_b", (b, E, d), seed, DEV, dtype)
    win = synth.draw("C_a", (b, n, d), seed, DEV, dtype)
    sink = synth.draw("sink", (H,), seed, DEV, "f32")
    qpos = np.stack([np.sort(rng.integers(0, n, size=T)) for _ in range(b)]).astype(np.int32)
    qpos[0, -1] = n - 1
    qpos[0, 0] = 0
    m = max(1, (n // E))
    if dense:
        idx_np = cnt_np = None
    else:
        idx_np = np.full((b, T, k), -1, np.int32)
        cnt_np = np.zeros((b, T), np.int32)
        for s in range(b):
            scr = rng.normal(size=(T, E))
            idx_np[s], cnt_np[s] = csa.topk(scr, qpos[s], m, k)
    return dict(q=q, kv=kv, win=win, sink=sink, qpos=qpos, idx=idx_np, cnt=cnt_np, m=m, tdt=tdt)


@pytest.mark.parametrize("H,d,k,n_w,dtype,dense,T,E,n,d_rope_out", [
    (64, 512, 512, 128, "bf16", False, 1, 1500, 6000, 0),   # decode shape, ragged
    (64, 512, 512, 128, "bf16", True, 1, 700, 2800, 0),     # HCA-style dense, E(t) up to 700
    (64, 512, 64, 128, "bf16", False, 9, 300, 1200, 0),     # prefill shape, several queries
    (4, 64, 16, 16, "f32", False, 40, 256, 1024, 0),        # tiny fp32
    # inverse RoPE on the output's last dims: cluster merge, workspace merge, one split, SIMT
    (64, 512, 512, 128, "bf16", False, 1, 1500, 6000, 64),
    (64, 512, 512, 128, "bf16", True, 1, 700, 2800, 64),
    (64, 512, 64, 128, "bf16", False, 9, 300, 1200, 64),
    (4, 64, 16, 16, "f32", False, 40, 256, 1024, 16),
])
def test_sparse_attention(H, d, k, n_w, dtype, dense, T, E, n, d_rope_out):
    b = 2
    c = _attn_case(b, T, H, d, E, n, k, n_w, dtype, dense, 51)
    scale = 1.0 / math.sqrt(d)
    out = torch.empty((b, T, H, d), dtype=c["tdt"], device=DEV)
    lse = torch.empty((b, T, H), dtype=torch.float32, device=DEV)
    p = L.AttnParams(H=H, d=d, n_w=n_w, scale=scale, m=c["m"], k=0 if dense else k,
                     dtype=L.DTYPE[dtype], d_rope_out=d_rope_out, rope_theta=1e4)
    wsb = L.csa_sparse_attn_workspace_size(p, b, T, E)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_sparse_attn(p, c["q"], c["kv"], E, _dev(c["idx"]), _dev(c["cnt"]), c["win"], n,
                      _dev(c["qpos"]), c["sink"], b, T, out, lse, ws, wsb)
    torch.cuda.synchronize()
    for s in range(b):
        o, l = csa.sparse_attn(f64(c["q"][s]), f64(c["kv"][s]),
                               None if dense else c["idx"][s], None if dense else c["cnt"][s],
                               f64(c["win"][s]), c["qpos"][s], f64(c["sink"]), n_w, scale, m=c["m"],
                               inv_rope=(d_rope_out, 1e4) if d_rope_out else None)
        if dtype == "bf16":
            assert_abs_close(f64(out[s]), o, 2e-2, "attention bf16")
        else:
            assert_rel_close(f64(out[s]), o, 1e-5, "attention f32")
        assert_abs_close(f64(lse[s]), l, 1e-3 * (1 + np.max(np.abs(l))), "lse")


@pytest.mark.parametrize("tile_of_spike", [1, 2])
def test_attention_lazy_rescale_path(tile_of_spike):
    """A row far above the first tile's maximum (in a later tile) forces the running-max
    update and the rescale of the accumulator; the result must still match the oracle."""
    b, T, H, d, E, n, k, n_w = 1, 3, 64, 512, 600, 2400, 256, 128
    c = _attn_case(b, T, H, d, E, n, k, n_w, "bf16", False, 61)
    qpos = c["qpos"]
    qpos[0, :] = [n - 1, n - 2, 1500]
    c["qpos"] = qpos
    rng = np.random.default_rng(5)
    for t in range(T):
        scr = rng.normal(size=(1, E))
        c["idx"][0, t], c["cnt"][0, t] = [a[0] for a in csa.topk(scr, qpos[0, t:t + 1], c["m"], k)]
    # plant: the selected entry at list position 128 * tile_of_spike + 5 is 30 x q[head 0] / |q|
    q0 = c["q"][0, 0, 0].float()
    pos = 128 * tile_of_spike + 5
    e = int(c["idx"][0, 0, pos]) if pos < k else None
    if e is None:
        u = int(qpos[0, 0]) - n_w + 1 + (pos - k)      # window token at list position pos
        c["win"][0, u] = (30 * q0 / q0.norm()).to(torch.bfloat16)
    else:
        c["kv"][0, e] = (30 * q0 / q0.norm()).to(torch.bfloat16)
    scale = 1.0 / math.sqrt(d)
    out = torch.empty((b, T, H, d), dtype=torch.bfloat16, device=DEV)
    p = L.AttnParams(H=H, d=d, n_w=n_w, scale=scale, m=c["m"], k=k, dtype=L.CSA_BF16)
    wsb = L.csa_sparse_attn_workspace_size(p, b, T, E)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_sparse_attn(p, c["q"], c["kv"], E, _dev(c["idx"]), _dev(c["cnt"]), c["win"], n,
                      _dev(c["qpos"]), c["sink"], b, T, out, None, ws, wsb)
    torch.cuda.synchronize()
    o, _ = csa.sparse_attn(f64(c["q"][0]), f64(c["kv"][0]), c["idx"][0], c["cnt"][0],
                           f64(c["win"][0]), c["qpos"][0], f64(c["sink"]), n_w, scale)
    assert_abs_close(f64(out[0]), o, 2e-2, "attention with rescale")
    assert L.csa_device_error() == 0
