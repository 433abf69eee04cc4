"""CSA2 on the GPU: the hierarchical (candidate-pool) indexer and the Reuse / Reindex modes
of the fused decode step, against the oracle.

Source: "DeepSeek Technical Reports", section CSA2 (Cross-Layer KV and Index
Reuse; Hierarchical Sparse Indexer).

Acceptance:
  * pool top-k, stage-isolated: bit-exact against the top-k of the GPU's own full
    indexer scores restricted to the pool (the gathered keys are scored with the
    same arithmetic), and within the tie band of the oracle's exact scores;
  * decode modes: the selection as above, attention max-abs 2e-2 against the oracle
    attention over the selection used.
"""

import math

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import runner, synth, workloads
from oracle import csa, pipeline

from helpers import assert_abs_close, f64
from test_gpu_stages import _dev, _index_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _pool_band_check(gi, gc, exact_pool_scores, pool_entries, k, rel_band=1e-3):
    """GPU selection vs the exact scores of the visible pool entries: equal except within the
    tie band of the k-th exact score."""
    from helpers import bf16_ulp
    n = len(pool_entries)
    assert gc == min(k, n)
    sel = list(gi[:gc])
    assert all(x == -1 for x in gi[gc:])
    assert sel == sorted(sel) and set(sel) <= set(pool_entries)
    if n <= k:
        return
    order = np.lexsort((pool_entries, -exact_pool_scores))
    ref = set(np.asarray(pool_entries)[order[:k]].tolist())
    tau = exact_pool_scores[order[k - 1]]
    band = max(rel_band * abs(tau), float(bf16_ulp(tau)))
    sc = dict(zip(np.asarray(pool_entries).tolist(), exact_pool_scores.tolist()))
    for e in ref.symmetric_difference(sel):
        assert abs(sc[e] - tau) <= band, (e, sc[e], tau)


@pytest.mark.parametrize("fmt,H,d,T", [("fp8", 64, 128, 1), ("nvfp4", 64, 128, 1),
                                        ("fp8", 64, 128, 3), ("f32", 4, 32, 2)])
def test_pool_topk_stage(fmt, H, d, T):
    b, E, m, P, k = 2, 3000, 4, 700, 64
    x = _index_inputs(b, T, E, H, d, fmt, 57)
    rng = np.random.default_rng(58)
    qpos = np.full((b, T), m * E - 1, dtype=np.int32)
    qpos[1, -1] = m * 1500 + 1                    # causal cut inside the pool
    pool = np.full((b, T, P), -1, dtype=np.int32)
    pcnt = np.zeros((b, T), dtype=np.int32)
    for s in range(b):
        for t in range(T):
            n = P if (s + t) % 2 == 0 else P - 111  # ragged pools, -1 padded
            pool[s, t, :n] = np.sort(rng.choice(E, size=n, replace=False))
            pcnt[s, t] = n
    pcnt[0, 0] = 50                               # fewer candidates than k
    p = L.IndexParams(H_I=H, d_I=d, m=m, qk_dtype=L.DTYPE[fmt], score_dtype=L.CSA_BF16)
    wsb = L.csa_pool_topk_workspace_size(p, b, T, P, k)
    ws = torch.full((wsb,), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    idx = torch.empty((b, T, k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((b, T), dtype=torch.int32, device=DEV)
    L.csa_pool_topk(p, _dev(x["q"]), _dev(x["qs"]), _dev(x["w"]), _dev(x["k"]), _dev(x["ks"]),
                    _dev(qpos), b, T, E, E, _dev(pool), _dev(pcnt), P, k, idx, cnt, ws)
    # the GPU's own full scores of the same codes
    full = torch.empty((b, T, E), dtype=torch.bfloat16, device=DEV)
    L.csa_index_scores(p, _dev(x["q"]), _dev(x["qs"]), _dev(x["w"]), _dev(x["k"]), _dev(x["ks"]),
                       _dev(qpos), b, T, E, E, full)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    gi, gc, gfull = idx.cpu().numpy(), cnt.cpu().numpy(), f64(full)
    for s in range(b):
        exact_all = csa.index_scores(x["qd"][s], x["w"][s], x["kd"][s], qpos[s], m, "f64")
        for t in range(T):
            ev = (qpos[s, t] + 1) // m
            cand = pool[s, t, :pcnt[s, t]]
            cand = cand[(cand >= 0) & (cand < min(ev, E))]
            # (1) bit-exact: top-k of the GPU's full scores over the visible pool
            order = np.lexsort((cand, -gfull[s, t, cand]))
            ref = np.sort(cand[order[:k]])
            assert gc[s, t] == len(ref)
            np.testing.assert_array_equal(gi[s, t, :gc[s, t]], ref)
            assert np.all(gi[s, t, gc[s, t]:] == -1)
            # (2) the oracle's exact scores: differences only inside the tie band
            _pool_band_check(gi[s, t], gc[s, t], exact_all[t, cand], cand, k)
            ri, rc = csa.pool_topk(x["qd"][s][t:t + 1], x["w"][s][t:t + 1], x["kd"][s],
                                   pool[s, t][None], pcnt[s, t:t + 1], qpos[s, t:t + 1], m, k)
            assert rc[0] == gc[s, t]


def _decode_in_mode(st, w, mode, P=0, **tensors):
    p = runner.decode_params(w, st.E_cap)
    p.mode, p.P = mode, P
    t = st.tensors(**{k: v for k, v in tensors.items() if k in ("q", "q_I", "w_")})
    t.update({k: v for k, v in tensors.items() if k in ("idx_in", "count_in", "pool",
                                                         "pool_count")})
    out = torch.empty_like(st.out)
    t["out"] = out
    idx = torch.full((w.b, w.k), -7, dtype=torch.int32, device=DEV)
    cnt = torch.full((w.b,), -7, dtype=torch.int32, device=DEV)
    t["idx_out"], t["count_out"] = idx, cnt
    wsb = L.csa_decode_workspace_size(p)
    ws = torch.empty((max(wsb, 256),), dtype=torch.uint8, device=DEV)
    L.csa_decode(p, t, ws, wsb)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    return out, idx, cnt


@pytest.mark.parametrize("base", ["64k_fp8", "1m_nvfp4"])
def test_decode_reuse_and_reindex_modes(base):
    w0 = workloads.CSA_DECODE_64K if base == "64k_fp8" else workloads.CSA_DECODE_1M
    w = workloads.shrink(w0, b=2, n=4 * 3000)
    inp = synth.make_inputs(w, device=DEV)
    st = runner.DecodeState(w, inp)
    st.build_caches()
    st.step()                                          # layer 1: full indexer, caches complete
    torch.cuda.synchronize()
    idx1 = st.idx.clone()
    cnt1 = st.count.clone()
    t = w.n - 1
    E = w.E
    # layer 2's own query heads, index query and weights
    q2 = synth.draw("q", tuple(inp["q"].shape), 91, DEV, w.dtype)
    qI2 = synth.draw("q_I", tuple(inp["q_I"].shape), 92, DEV, w.dtype)
    w2 = synth.draw("w", tuple(inp["w"].shape), 93, DEV, "f32", dist="uniform", spread=1 / 64)
    # Reuse: layer 1's selection with layer 2's q
    out_r, idx_r, cnt_r = _decode_in_mode(st, w, L.CSA_MODE_REUSE, q=q2, idx_in=idx1,
                                          count_in=cnt1)
    assert torch.all(idx_r == -7)                      # no selection written in Reuse mode
    # Reindex: the pool is layer 1's top-P (P = 2k) of its own scores
    P = 2 * w.k
    ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                       score_dtype=L.CSA_BF16)
    codes = torch.empty((w.b * w.H_I, runner.row_bytes(w.idx_dtype, w.c_I)), dtype=torch.uint8,
                        device=DEV)
    qs = torch.empty((w.b * w.H_I,), dtype=torch.float32, device=DEV) if w.idx_dtype == "fp8" \
        else torch.empty((w.b * w.H_I, w.c_I // 16), dtype=torch.uint8, device=DEV)
    L.csa_quantize(L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], inp["q_I"], w.b * w.H_I, w.c_I, codes,
                   qs)
    qpos = torch.full((w.b, 1), t, dtype=torch.int32, device=DEV)
    sc1 = torch.empty((w.b, 1, E), dtype=torch.bfloat16, device=DEV)
    L.csa_index_scores(ip, codes, qs, inp["w"], st.kI_cache, st.kI_scales, qpos, w.b, 1, st.E_cap,
                       E, sc1)
    pool = torch.empty((w.b, 1, P), dtype=torch.int32, device=DEV)
    pcnt = torch.empty((w.b, 1), dtype=torch.int32, device=DEV)
    tkb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, 1, E, P)
    tkws = torch.empty((max(tkb, 256),), dtype=torch.uint8, device=DEV)
    L.csa_topk(sc1, L.CSA_BF16, qpos, w.m, w.b, 1, E, P, pool, pcnt, tkws, tkb)
    out_x, idx_x, cnt_x = _decode_in_mode(st, w, L.CSA_MODE_REINDEX, P=P, q=q2, q_I=qI2, w_=w2,
                                          pool=pool.reshape(w.b, P), pool_count=pcnt.reshape(w.b))
    for s in range(w.b):
        g = {k: f64(v[s]) for k, v in inp.items() if v.dim() >= 3}
        main = dict(C_a=g["C_a"], Z_a=g["Z_a"], B_a=f64(inp["B_a"]), C_b=g["C_b"], Z_b=g["Z_b"],
                    B_b=f64(inp["B_b"]))
        index = dict(C_a=g["CI_a"], Z_a=g["ZI_a"], B_a=f64(inp["BI_a"]), C_b=g["CI_b"],
                     Z_b=g["ZI_b"], B_b=f64(inp["BI_b"]))
        sink = f64(inp["sink"])
        kw = dict(L=w.n, m=w.m, d_rope=w.d_rope, theta=w.theta, eps=w.eps, k=w.k, n_w=w.n_w,
                  scale=w.scale, kv_dtype=w.dtype, idx_dtype=w.idx_dtype)

        def attend(sel, q):
            kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                          main["Z_b"], main["B_b"], w.m, True, sel, w.d_rope,
                                          w.theta, w.eps)
            rows = np.concatenate([pipeline.round_out(kv_sel, w.dtype),
                                   main["C_a"][csa.window_rows(t, w.n_w)]])
            return csa.attend(q, rows, sink, w.scale)[0]

        # Reuse: exactly layer 1's rows with layer 2's q
        sel1 = idx1[s, :int(cnt1[s])].cpu().numpy().astype(np.int64)
        q2s = f64(q2[s, 0])
        assert_abs_close(f64(out_r[s]), attend(sel1, q2s), 2e-2, "reuse attention")
        ref = pipeline.csa_decode_seq(main, index, q2s, f64(qI2[s, 0]), f64(w2[s, 0]), sink,
                                      mode="reuse", idx_in=idx1[s].cpu().numpy(), **kw)
        assert_abs_close(f64(out_r[s]), ref["out"], 2e-2, "reuse vs oracle composition")
        # Reindex: the pool's best k under layer 2's index query
        pl = pool[s, 0, :int(pcnt[s, 0])].cpu().numpy().astype(np.int64)
        qd2 = pipeline.quantize_rows(f64(qI2[s, 0])[None], w.idx_dtype)[0]
        kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                index["Z_b"], index["B_b"], w.m, True, 0, E, w.d_rope_I, w.theta,
                                w.eps)
        kd = pipeline.quantize_rows(kI, w.idx_dtype)[0]
        exact = csa.index_scores(qd2, f64(w2[s, 0])[None], kd[pl], np.array([t]), w.m, "f64")[0]
        gi = idx_x[s].cpu().numpy()
        gc = int(cnt_x[s])
        _pool_band_check(gi, gc, exact, pl, w.k)
        sel = gi[:gc].astype(np.int64)
        assert_abs_close(f64(out_x[s]), attend(sel, q2s), 2e-2, "reindex attention")
        ref = pipeline.csa_decode_seq(main, index, q2s, f64(qI2[s, 0]), f64(w2[s, 0]), sink,
                                      mode="reindex", pool=pool[s, 0].cpu().numpy(), **kw)
        if np.array_equal(gi, ref["idx"]):
            assert_abs_close(f64(out_x[s]), ref["out"], 2e-2, "reindex vs oracle composition")
        else:
            assert_abs_close(f64(out_x[s]), ref["out"], 5e-2, "reindex vs oracle selection")
