"""End-to-end parity of the fused drivers (csa_prefill / csa_decode) against the oracle.

The tiny fp32 prefill runs in full; the decode and 32K-prefill workloads run
here at reduced context (same dims, types and tile structure, ragged where the
shape allows); ``test_gpu_fullsize.py`` covers the full sizes on samples.

Acceptance per stage:
  compressed entries: relative 1e-5 (float32 storage) / 2e-2 (bf16 storage);
  top-k: exact, except entries whose exact score sits within the tie band
         (max(1e-3 |tau|, one bf16 ulp of tau)) of the k-th score tau;
  attention: max-abs 2e-2 (bf16) / relative 1e-5 (float32) on the oracle's
         selection; where the GPU chose a different (valid) set, the output is
         re-checked against the oracle attention over the GPU's set at the same
         tolerance, and against the oracle's own output at 5e-2.
"""

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import runner, synth, workloads
from oracle import csa, pipeline

from helpers import assert_abs_close, assert_rel_close, f64, topk_band_check

pytestmark = pytest.mark.gpu


def _np(inp, s=None):
    out = {}
    for k, v in inp.items():
        out[k] = f64(v[s]) if (s is not None and v.dim() >= 3) or (s is not None and k == "w") else f64(v)
    return out


def _branches(g):
    main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g.get("C_b"), Z_b=g.get("Z_b"),
                B_b=g.get("B_b"))
    index = dict(C_a=g.get("CI_a"), Z_a=g.get("ZI_a"), B_a=g.get("BI_a"), C_b=g.get("CI_b"),
                 Z_b=g.get("ZI_b"), B_b=g.get("BI_b"))
    return main, index


def _check_attention(w, gpu_out, ref_out, same_sel, recheck, atol_bf16=2e-2):
    if w.dtype == "f32":
        if same_sel:
            assert_rel_close(gpu_out, ref_out, 1e-5, "attention f32")
        else:
            assert_rel_close(gpu_out, recheck(), 1e-5, "attention f32 on the GPU's selection")
    else:
        if same_sel:
            assert_abs_close(gpu_out, ref_out, atol_bf16, "attention")
        else:
            assert_abs_close(gpu_out, recheck(), atol_bf16, "attention on the GPU's selection")
            assert_abs_close(gpu_out, ref_out, 5e-2, "attention vs oracle selection")


@pytest.mark.parametrize("inv_rope", [False, True])
def test_tiny_prefill_f32_full(inv_rope):
    w = workloads.shrink(workloads.TINY, inv_rope=inv_rope)
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PrefillState(w, inp)
    st.run()
    torch.cuda.synchronize()
    g = _np(inp, 0)
    main, index = _branches(g)
    ref = pipeline.csa_prefill(main, index, g["q"], g["q_I"], g["w"], g["sink"], m=w.m,
                               d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k, n_w=w.n_w,
                               scale=w.scale, kv_dtype="f32", idx_dtype="f32", score_dtype="f32",
                               inv_rope=w.inv_rope)
    assert_rel_close(f64(st.kv_cache[0]), ref["kv"], 1e-5, "kv cache")
    assert_rel_close(f64(st.kI_cache[0]), ref["kI"], 1e-5, "index keys")
    exact = csa.index_scores(ref["qI_deq"], g["w"], ref["kI_deq"], np.arange(w.n), w.m, "f64")
    gi = st.idx[0].cpu().numpy()
    gc = st.count[0].cpu().numpy()
    out = f64(st.out[0])
    nd = 0
    for t in range(w.n):
        ev = (t + 1) // w.m
        nd += topk_band_check(gi[t], gc[t], exact[t], ev, w.k)
        same = np.array_equal(gi[t], ref["idx"][t])

        def recheck(t=t):
            o, _ = csa.sparse_attn(g["q"][t:t + 1], ref["kv_stored"], gi[t:t + 1], gc[t:t + 1],
                                   g["C_a"], [t], g["sink"], w.n_w, w.scale,
                                   inv_rope=(w.d_rope, w.theta) if w.inv_rope else None)
            return o[0]
        _check_attention(w, out[t], ref["out"][t], same, recheck)
    assert nd <= 2, nd
    assert_abs_close(f64(st.lse[0]), ref["lse"], 1e-4, "lse")


def _decode_case(w, seqs):
    inp = synth.make_inputs(w, device="cuda")
    st = runner.DecodeState(w, inp)
    st.build_caches()
    st.step()
    torch.cuda.synchronize()
    t = w.n - 1
    for s in seqs:
        g = _np(inp, s)
        main, index = _branches(g)
        q = g["q"][0]
        if w.kind == "hca_decode":
            ref = pipeline.hca_decode_seq(main, q, g["sink"], L=w.n, m=w.m, d_rope=w.d_rope,
                                          theta=w.theta, eps=w.eps, n_w=w.n_w, scale=w.scale,
                                          kv_dtype=w.dtype, inv_rope=w.inv_rope)
            assert_rel_close(f64(st.kv_cache[s]), ref["kv"], 2e-2, "hca cache (incl. new entry)")
            assert_abs_close(f64(st.out[s]), ref["out"], 2e-2, "hca attention")
            continue
        ref = pipeline.csa_decode_seq(main, index, q, g["q_I"][0], g["w"][0], g["sink"], L=w.n,
                                      m=w.m, d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k,
                                      n_w=w.n_w, scale=w.scale, kv_dtype=w.dtype,
                                      idx_dtype=w.idx_dtype, inv_rope=w.inv_rope)
        E = w.E
        assert_rel_close(f64(st.kv_cache[s, E - 1]), ref["new_entry"], 2e-2, "new latent entry")
        exact = csa.index_scores(ref["qI_deq"], g["w"][0][None], ref["kI_deq"], np.array([t]),
                                 w.m, "f64")[0]
        gi = st.idx[s].cpu().numpy()
        gc = int(st.count[s].cpu())
        topk_band_check(gi, gc, exact, E, w.k)   # the acceptance: differences only inside the tie band
        same = np.array_equal(gi, ref["idx"])

        def recheck():
            sel = gi[:gc].astype(np.int64)
            kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                          main["Z_b"], main["B_b"], w.m, True, sel, w.d_rope,
                                          w.theta, w.eps)
            rows = np.concatenate([pipeline.round_out(kv_sel, w.dtype),
                                   main["C_a"][csa.window_rows(t, w.n_w)]])
            o = csa.attend(q, rows, g["sink"], w.scale)[0]
            return csa.inverse_rope(o, t, w.d_rope, w.theta) if w.inv_rope else o
        _check_attention(w, f64(st.out[s]), ref["out"], same, recheck)


@pytest.mark.parametrize("inv_rope", [False, True])
def test_csa_decode_fp8_small(inv_rope):
    w = workloads.shrink(workloads.CSA_DECODE_64K, b=3, n=4100 - 4100 % 4,   # E = 1025: ragged tile
                         inv_rope=inv_rope)
    _decode_case(w, [0, 2])


def test_csa_decode_nvfp4_small():
    w = workloads.shrink(workloads.CSA_DECODE_1M, b=2, n=4 * 3000)
    _decode_case(w, [1])


@pytest.mark.parametrize("inv_rope", [False, True])
def test_hca_decode_small(inv_rope):
    w = workloads.shrink(workloads.HCA_DECODE_1M, b=2, n=128 * 70, inv_rope=inv_rope)
    _decode_case(w, [0, 1])


def test_csa_decode_short_context():
    """Context shorter than k entries: top-k keeps everything (E(t) <= k)."""
    w = workloads.shrink(workloads.CSA_DECODE_64K, b=2, n=4 * 300)
    _decode_case(w, [0])


def test_csa_prefill_fp8_sampled():
    w = workloads.shrink(workloads.CSA_PREFILL_32K, n=4096)
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PrefillState(w, inp)
    st.run()
    torch.cuda.synchronize()
    rng = np.random.default_rng(3)
    rows = np.unique(np.concatenate([[0, 1, 2, 3, 4, 127, 128, 2046, 2047, 2048, 4095],
                                     rng.integers(0, w.n, 24)]))
    g = _np(inp, 0)
    main, index = _branches(g)
    ref = pipeline.csa_prefill(main, index, g["q"], g["q_I"], g["w"], g["sink"], m=w.m,
                               d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k, n_w=w.n_w,
                               scale=w.scale, kv_dtype="bf16", idx_dtype="fp8", score_dtype="bf16",
                               query_rows=rows)
    assert_rel_close(f64(st.kv_cache[0]), ref["kv"], 2e-2, "kv cache")
    exact = csa.index_scores(ref["qI_deq"], g["w"][rows], ref["kI_deq"], rows, w.m, "f64")
    gi = st.idx[0].cpu().numpy()
    gc = st.count[0].cpu().numpy()
    out = f64(st.out[0])
    nd = 0
    for j, t in enumerate(rows):
        ev = (t + 1) // w.m
        nd += topk_band_check(gi[t], gc[t], exact[j], ev, w.k)
        same = np.array_equal(gi[t], ref["idx"][j])

        def recheck(t=t):
            o, _ = csa.sparse_attn(g["q"][t:t + 1], ref["kv_stored"], gi[t:t + 1], gc[t:t + 1],
                                   g["C_a"], [t], g["sink"], w.n_w, w.scale)
            return o[0]
        _check_attention(w, out[t], ref["out"][j], same, recheck)


@pytest.mark.parametrize("fmt,paged", [("fp8", False), ("fp8", True), ("nvfp4", False)])
def test_fused_decode_selection_equals_stage_calls(fmt, paged):
    """The fused decode quantises the bf16 index queries with the arithmetic of
    csa_quantize (FP8: inside the indexer, so that only the key page the step writes waits
    for the compressor; NVFP4: in the prologue): the selection is bit for bit the one of
    the stage calls (csa_quantize, csa_index_scores, csa_topk) on the updated cache."""
    from long_context_sparse_05_b200 import _lib as L
    base = workloads.CSA_DECODE_64K if fmt == "fp8" else workloads.CSA_DECODE_1M
    w = workloads.shrink(base, b=3, n=4100 - 4100 % 4)
    inp = synth.make_inputs(w, device="cuda")
    E = w.E
    if paged:
        st = runner.PagedDecodeState(w, inp, shuffle_seed=9)
        st.step()
        # each sequence's key rows in entry order, gathered from its pages (FP8 scales are
        # one float per row)
        e = torch.arange(E, device="cuda")
        PE = L.PAGE_ENTRIES
        rows = st.block_table[:, e // PE].long() * PE + e % PE
        E_cap = (E + 3) // 4 * 4
        kI = torch.zeros((w.b, E_cap, w.c_I), dtype=torch.uint8, device="cuda")
        kI[:, :E] = st.kI_pages[rows]
        ks = torch.zeros((w.b, E_cap), dtype=torch.float32, device="cuda")
        ks[:, :E] = st.kI_scales[rows]
    else:
        st = runner.DecodeState(w, inp)
        st.build_caches()
        st.step()
        kI, ks, E_cap = st.kI_cache, st.kI_scales, st.E_cap
    torch.cuda.synchronize()
    rows_q = w.b * w.H_I
    codes = torch.empty((rows_q, runner.row_bytes(fmt, w.c_I)), dtype=torch.uint8, device="cuda")
    sc = (torch.empty((rows_q,), dtype=torch.float32, device="cuda") if fmt == "fp8" else
          torch.empty((rows_q, w.c_I // 16), dtype=torch.uint8, device="cuda"))
    L.csa_quantize(L.CSA_BF16, L.DTYPE[fmt], inp["q_I"], rows_q, w.c_I, codes, sc)
    qpos = torch.full((w.b, 1), w.n - 1, dtype=torch.int32, device="cuda")
    ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[fmt], score_dtype=L.CSA_BF16)
    scores = torch.empty((w.b, 1, E), dtype=torch.bfloat16, device="cuda")
    L.csa_index_scores(ip, codes, sc, inp["w"], kI, ks, qpos, w.b, 1, E_cap, E, scores)
    idx = torch.empty((w.b, 1, w.k), dtype=torch.int32, device="cuda")
    cnt = torch.empty((w.b, 1), dtype=torch.int32, device="cuda")
    wsb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, 1, E, w.k)
    ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device="cuda")
    L.csa_topk(scores, L.CSA_BF16, qpos, w.m, w.b, 1, E, w.k, idx, cnt, ws, wsb)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    assert torch.equal(cnt.view(-1), st.count.view(-1))
    assert torch.equal(idx.view(w.b, -1), st.idx.view(w.b, -1))
