"""The paged decode step (csa_decode_paged) against the oracle: classical caches in pages
behind a shuffled block table, a per-sequence state of window and raw tail rows, and
sequences of a batch at different positions (in-block and block-completing tokens).

Source: "DeepSeek-V4技术报告解读", section 3.2 (异构 KV 缓存管理: classical KV cache in
blocks per request; state cache of the sliding window and the not yet compressed tail).

Acceptance: as the whole-sequence decode step (test_gpu_e2e.py): the new entry within
2e-2 relative of the oracle's (bf16 storage); selections equal except inside the tie
band; attention max-abs 2e-2 on the selection used; the state rings hold the new rows.
"""

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import runner, synth, workloads
from oracle import csa, pipeline

from helpers import assert_abs_close, assert_rel_close, f64, topk_band_check

pytestmark = pytest.mark.gpu


def _seq(inp, s):
    return {k: (f64(v[s]) if v.dim() >= 3 else f64(v)) for k, v in inp.items()}


def _check(w, st, inp):
    m = w.m
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    for s, t in enumerate(st.positions):
        g = _seq(inp, s)
        main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=g["B_a"], C_b=g.get("C_b"), Z_b=g.get("Z_b"),
                    B_b=g.get("B_b"))
        q = g["q"][0]
        if st.hca:
            ref = pipeline.hca_decode_at(main, q, g["sink"], t=t, m=m, d_rope=w.d_rope,
                                         theta=w.theta, eps=w.eps, n_w=w.n_w, scale=w.scale,
                                         kv_dtype=w.dtype, inv_rope=w.inv_rope)
            assert_abs_close(f64(st.out[s]), ref["out"], 2e-2, "paged hca attention")
        else:
            index = dict(C_a=g["CI_a"], Z_a=g["ZI_a"], B_a=g["BI_a"], C_b=g["CI_b"],
                         Z_b=g["ZI_b"], B_b=g["BI_b"])
            ref = pipeline.csa_decode_at(main, index, q, g["q_I"][0], g["w"][0], g["sink"], t=t,
                                         m=m, d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k,
                                         n_w=w.n_w, scale=w.scale, kv_dtype=w.dtype,
                                         idx_dtype=w.idx_dtype, inv_rope=w.inv_rope)
            Et = (t + 1) // m
            gi = st.idx[s].cpu().numpy()
            gc = int(st.count[s])
            if Et > 0:
                kd = pipeline.quantize_rows(ref["kI"], w.idx_dtype)[0]
                qd = pipeline.quantize_rows(g["q_I"][0][None], w.idx_dtype)[0]
                exact = csa.index_scores(qd, g["w"][0][None], kd, np.array([t]), m, "f64")[0]
                topk_band_check(gi, gc, exact, Et, w.k)
            else:
                assert gc == 0
            sel = gi[:gc].astype(np.int64)
            kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                          main["Z_b"], main["B_b"], m, True, sel, w.d_rope,
                                          w.theta, w.eps)
            rows = np.concatenate([pipeline.round_out(kv_sel, w.dtype).reshape(-1, w.c),
                                   main["C_a"][csa.window_rows(t, w.n_w)]])
            o = csa.attend(q, rows, g["sink"], w.scale)[0]
            if w.inv_rope:
                o = csa.inverse_rope(o, t, w.d_rope, w.theta)
            assert_abs_close(f64(st.out[s]), o, 2e-2, "paged attention on the GPU's selection")
            if np.array_equal(gi, ref["idx"]):
                assert_abs_close(f64(st.out[s]), ref["out"], 2e-2, "paged attention")
        # the entry the token completes, in its page
        if (t + 1) % m == 0:
            row = st.entry_row(s, (t + 1) // m - 1)
            assert_rel_close(f64(st.kv_pages[row]), ref["new_entry"], 2e-2, "new entry in its page")
        # the state now holds the new token's rows
        R = st.ring
        assert torch.equal(st.tails["tail_C_a"][s, t % R], inp["C_a"][s, t])
        assert torch.equal(st.tails["tail_Z_a"][s, t % R], inp["Z_a"][s, t])
        if not st.hca:
            assert torch.equal(st.tails["tail_C_b"][s, t % R], inp["C_b"][s, t])
            assert torch.equal(st.tails["tail_ZI_b"][s, t % R], inp["ZI_b"][s, t])
        assert torch.equal(st.win[s, t % w.n_w], inp["C_a"][s, t])


@pytest.mark.parametrize("base,inv_rope", [("64k_fp8", False), ("1m_nvfp4", True)])
def test_paged_csa_decode_variable_lengths(base, inv_rope):
    w0 = workloads.CSA_DECODE_64K if base == "64k_fp8" else workloads.CSA_DECODE_1M
    n = 4 * 1400
    w = workloads.shrink(w0, b=5, n=n, inv_rope=inv_rope)
    # block-completing, in-block, a short context (E(t) < k), one shorter than a block
    positions = [n - 1, n - 3, 4 * 700 + 1, 4 * 130 - 1, 2]
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PagedDecodeState(w, inp, positions=positions, shuffle_seed=3)
    st.step()
    _check(w, st, inp)


def test_paged_hca_decode_variable_lengths():
    n = 128 * 600
    w = workloads.shrink(workloads.HCA_DECODE_1M, b=3, n=n)
    positions = [n - 1, 128 * 300 + 17, 100]
    inp = synth.make_inputs(w, device="cuda")
    st = runner.PagedDecodeState(w, inp, positions=positions, shuffle_seed=4)
    st.step()
    _check(w, st, inp)


def test_paged_equals_whole_sequence_decode():
    """All sequences at the last token of a whole context: the paged step gives the same
    output as csa_decode on the same inputs (the same kernels, different addressing)."""
    w = workloads.shrink(workloads.CSA_DECODE_64K, b=3, n=4 * 1500)
    inp = synth.make_inputs(w, device="cuda")
    a = runner.DecodeState(w, inp)
    a.build_caches()
    a.step()
    bst = runner.PagedDecodeState(w, inp, shuffle_seed=5)
    bst.step()
    torch.cuda.synchronize()
    assert torch.equal(a.idx, bst.idx)
    assert torch.equal(a.out, bst.out)
