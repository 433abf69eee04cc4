"""Parity at the full sizes the benchmark runs, on sampled outputs.

Each workload runs exactly as bench.py runs it (same shapes, seeds, launch
configuration); the oracle recomputes, from the raw inputs, the outputs of
sampled sequences (decode) or sampled query rows (prefill), reading the device
inputs row by row (``LazyRows``).  Acceptance is as in test_gpu_e2e.py.
"""

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import runner, synth, workloads
from oracle import csa, pipeline

from helpers import LazyRows, assert_abs_close, assert_rel_close, f64, topk_band_check

pytestmark = pytest.mark.gpu


def _seq(inp, s):
    """One sequence of the inputs: big tensors lazily, small ones as float64 arrays."""
    out = {}
    for k, v in inp.items():
        if v.dim() >= 3:
            out[k] = LazyRows(v[s]) if v.shape[1] > 4096 else f64(v[s])
        else:
            out[k] = f64(v)
    return out


def _branches(g):
    main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g.get("C_b"), Z_b=g.get("Z_b"),
                B_b=g.get("B_b"))
    index = dict(C_a=g.get("CI_a"), Z_a=g.get("ZI_a"), B_a=g.get("BI_a"), C_b=g.get("CI_b"),
                 Z_b=g.get("ZI_b"), B_b=g.get("BI_b"))
    return main, index


def _csa_decode_full(w, seqs):
    inp = synth.make_inputs(w, device="cuda")
    st = runner.DecodeState(w, inp)
    st.build_caches()
    st.step()
    torch.cuda.synchronize()
    t = w.n - 1
    for s in seqs:
        g = _seq(inp, s)
        main, index = _branches(g)
        ref = pipeline.csa_decode_seq(main, index, g["q"][0], g["q_I"][0], g["w"][0], g["sink"],
                                      L=w.n, m=w.m, d_rope=w.d_rope, theta=w.theta, eps=w.eps,
                                      k=w.k, n_w=w.n_w, scale=w.scale, kv_dtype=w.dtype,
                                      idx_dtype=w.idx_dtype)
        E = w.E
        assert_rel_close(f64(st.kv_cache[s, E - 1]), ref["new_entry"], 2e-2, "new latent entry")
        # cache entries built by the compressor before the step: a seeded sample
        rng = np.random.default_rng(s)
        sample = np.unique(np.concatenate([[0, 1, E - 2], rng.integers(0, E - 1, 16)]))
        kv_ref = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                      main["Z_b"], main["B_b"], w.m, True, sample, w.d_rope,
                                      w.theta, w.eps)
        assert_rel_close(f64(st.kv_cache[s][torch.from_numpy(sample).cuda()]), kv_ref, 2e-2,
                         "cache sample")
        exact = csa.index_scores(ref["qI_deq"], g["w"][0][None], ref["kI_deq"], np.array([t]),
                                 w.m, "f64")[0]
        gi = st.idx[s].cpu().numpy()
        gc = int(st.count[s].cpu())
        topk_band_check(gi, gc, exact, E, w.k)   # the acceptance: differences only inside the tie band
        if np.array_equal(gi, ref["idx"]):
            assert_abs_close(f64(st.out[s]), ref["out"], 2e-2, "attention")
        else:
            sel = gi[:gc].astype(np.int64)
            kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                          main["Z_b"], main["B_b"], w.m, True, sel, w.d_rope,
                                          w.theta, w.eps)
            rows = np.concatenate([pipeline.round_out(kv_sel, w.dtype),
                                   main["C_a"][csa.window_rows(t, w.n_w)]])
            o, _ = csa.attend(g["q"][0], rows, g["sink"], w.scale)
            assert_abs_close(f64(st.out[s]), o, 2e-2, "attention on the GPU's selection")
            assert_abs_close(f64(st.out[s]), ref["out"], 5e-2, "attention vs oracle selection")
    del st, inp
    torch.cuda.empty_cache()


def test_csa_decode_64k_fp8_full():
    _csa_decode_full(workloads.CSA_DECODE_64K, [0, 11])


def test_csa_decode_1m_nvfp4_full():
    _csa_decode_full(workloads.CSA_DECODE_1M, [2])


def test_hca_decode_1m_full():
    w = workloads.HCA_DECODE_1M
    inp = synth.make_inputs(w, device="cuda")
    st = runner.DecodeState(w, inp)
    st.build_caches()
    st.step()
    torch.cuda.synchronize()
    for s in (5,):
        g = _seq(inp, s)
        main, _ = _branches(g)
        ref = pipeline.hca_decode_seq(main, g["q"][0], g["sink"], L=w.n, m=w.m, d_rope=w.d_rope,
                                      theta=w.theta, eps=w.eps, n_w=w.n_w, scale=w.scale,
                                      kv_dtype=w.dtype)
        assert_rel_close(f64(st.kv_cache[s]), ref["kv"], 2e-2, "HCA cache and new entry")
        assert_abs_close(f64(st.out[s]), ref["out"], 2e-2, "HCA attention")
    del st, inp
    torch.cuda.empty_cache()


def test_csa_prefill_32k_fp8_full_sampled():
    w = workloads.CSA_PREFILL_32K
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PrefillState(w, inp)
    st.run()
    torch.cuda.synchronize()
    rng = np.random.default_rng(8)
    rows = np.unique(np.concatenate([[0, 2, 3, 4, 127, 128, 2046, 2047, 2048, 32767],
                                     rng.integers(0, w.n, 6)]))
    g = _seq(inp, 0)
    main, index = _branches(g)
    ref = pipeline.csa_prefill(main, index, g["q"], g["q_I"], g["w"], g["sink"], m=w.m,
                               d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k, n_w=w.n_w,
                               scale=w.scale, kv_dtype="bf16", idx_dtype="fp8",
                               score_dtype="bf16", query_rows=rows)
    assert_rel_close(f64(st.kv_cache[0]), ref["kv"], 2e-2, "kv cache")
    exact = csa.index_scores(ref["qI_deq"], g["w"][rows], ref["kI_deq"], rows, w.m, "f64")
    gi = st.idx[0].cpu().numpy()
    gc = st.count[0].cpu().numpy()
    out = st.out[0]
    for j, t in enumerate(rows):
        ev = (t + 1) // w.m
        topk_band_check(gi[t], gc[t], exact[j], ev, w.k)
        if np.array_equal(gi[t], ref["idx"][j]):
            assert_abs_close(f64(out[t]), ref["out"][j], 2e-2, "attention row %d" % t)
        else:
            o, _ = csa.sparse_attn(g["q"][t:t + 1], ref["kv_stored"], gi[t:t + 1], gc[t:t + 1],
                                   main["C_a"], [t], g["sink"], w.n_w, w.scale)
            assert_abs_close(f64(out[t]), o[0], 2e-2, "attention row %d (GPU selection)" % t)
    del st, inp
    torch.cuda.empty_cache()
