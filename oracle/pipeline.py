"""Whole-path compositions of the oracle: CSA prefill, CSA decode step, HCA decode step.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).

The order of the stages is the operator graph of "DeepSeek V4 结构速览",
section "CSA（c4a 路线）": compressor -> (index-key compressor + quantiser) ->
lightning indexer -> top-k -> concatenation with the raw sliding window ->
shared-latent MQA with sink.  HCA (section "HCA（c128a 路线）") drops the
indexer and attends to every visible entry.

Every argument is a numpy array holding the values the caller feeds the
library (bf16 inputs given as float64 on the bf16 grid).  ``idx_dtype`` picks
the index-path number format: "f32" (no quantisation), "fp8" (E4M3, one fp32
scale per row of d_I) or "nvfp4" (E2M1, one UE4M3 scale per 16 elements).
"""

import numpy as np

from . import codecs
from . import csa


def round_out(x, dtype):
    """Round float64 results to the library's storage type ("bf16" or "f32")."""
    if dtype == "bf16":
        return codecs.round_to_bf16(x)
    if dtype == "f32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    raise ValueError(dtype)


def quantize_rows(x, idx_dtype):
    """Quantise rows (last axis) of the index path and return the dequantised float64 values.

    The quantiser consumes float32 values (the compressor's output precision),
    so the float64 input is first rounded to float32.
    Returns (dequantised values, raw pieces tuple).
    """
    x32 = np.asarray(x, dtype=np.float64).astype(np.float32)
    if idx_dtype == "f32":
        return x32.astype(np.float64), (x32,)
    if idx_dtype == "fp8":
        codes, scales = codecs.quant_fp8_rows(x32)
        return codecs.dequant_fp8_rows(codes, scales), (codes, scales)
    if idx_dtype == "nvfp4":
        packed, sc = codecs.quant_nvfp4(x32)
        return codecs.dequant_nvfp4(packed, sc), (packed, sc)
    raise ValueError(idx_dtype)


def csa_prefill(main, index, q, q_I, w, sink, *, m, d_rope, theta, eps, k, n_w, scale,
                kv_dtype, idx_dtype, score_dtype, query_rows=None, inv_rope=False):
    """CSA prefill of one sequence: every token t = 0..n-1 is a query.

    main / index: dicts with C_a, Z_a, B_a, C_b, Z_b, B_b ([n][c], [m][c]).
    q [n][H][d]; q_I [n][H_I][d_I] (unquantised); w [n][H_I]; sink [H].
    The raw window rows are the main branch's C_a (the uncompressed latent).
    ``query_rows`` restricts the queries evaluated (all entries are still
    compressed, as every query may select any visible entry).  ``inv_rope``
    applies ``csa.inverse_rope`` (the last d_rope dims) to every output.
    Returns a dict of every intermediate.
    """
    n = main["C_a"].shape[0]
    E = n // m
    kv = csa.compress_range(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                            main["B_b"], m, True, 0, E, d_rope, theta, eps)
    kv_st = round_out(kv, kv_dtype)
    kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"], index["Z_b"],
                            index["B_b"], m, True, 0, E, d_rope, theta, eps)
    kI_deq, _ = quantize_rows(kI, idx_dtype)
    rows = np.arange(n) if query_rows is None else np.asarray(query_rows, dtype=np.int64)
    qI_deq, _ = quantize_rows(q_I[rows], idx_dtype)
    scores = csa.index_scores(qI_deq, w[rows], kI_deq, rows, m, score_dtype)
    idx, cnt = csa.topk(scores, rows, m, k)
    o, lse = csa.sparse_attn(q[rows], kv_st, idx, cnt, main["C_a"], rows, sink, n_w, scale,
                             inv_rope=(d_rope, theta) if inv_rope else None)
    return dict(kv=kv, kv_stored=kv_st, kI=kI, kI_deq=kI_deq, qI_deq=qI_deq, scores=scores,
                idx=idx, cnt=cnt, out=round_out(o, kv_dtype), out_f64=o, lse=lse, rows=rows)


def csa_decode_seq(main, index, q, q_I, w, sink, *, L, m, d_rope, theta, eps, k, n_w, scale,
                   kv_dtype, idx_dtype, mode="full", idx_in=None, pool=None, inv_rope=False):
    """One CSA decode step of one sequence with L tokens of context.

    The new token is t = L - 1; it completes block E - 1 (E = L / m), so the
    step compresses that entry (main and index branch) and then scores all E
    entries, selects k of them and attends over them plus the window.  The
    earlier entries of the caches are the compressor's outputs for their own
    blocks (the state the decode step reads), computed here the same way.
    q [H][d]; q_I [H_I][d_I]; w [H_I].

    ``mode`` follows the operating modes of "DeepSeek Technical Reports",
    section CSA2 (cross-layer KV and index reuse):
      "full"    the indexer scores all E entries (the default above);
      "reuse"   no scoring: the selection ``idx_in`` (entry ids, -1 padded) of an
                earlier layer is attended with this layer's q;
      "reindex" hierarchical indexer: only the entries of ``pool`` (entry ids,
                -1 padded) are scored with this layer's q_I, and k kept
                (``csa.pool_topk``).
    ``inv_rope`` applies ``csa.inverse_rope`` (the last d_rope dims) to the output.
    """
    E = L // m
    t = L - 1
    kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"], index["Z_b"],
                            index["B_b"], m, True, 0, E, d_rope, theta, eps, chunk_rows=1 << 16)
    kI_deq, _ = quantize_rows(kI, idx_dtype)
    qI_deq, _ = quantize_rows(np.asarray(q_I)[None], idx_dtype)
    scores = csa.index_scores(qI_deq, np.asarray(w)[None], kI_deq, np.array([t]), m, "bf16")
    if mode == "full":
        idx, cnt = csa.topk(scores, np.array([t]), m, k)
    elif mode == "reuse":
        sel_in = np.asarray(idx_in).reshape(-1)
        idx = np.full((1, k), -1, dtype=np.int32)
        n_in = int(np.sum(sel_in >= 0))
        idx[0, :n_in] = sel_in[:n_in]
        cnt = np.array([n_in], dtype=np.int32)
    elif mode == "reindex":
        pl = np.asarray(pool).reshape(1, -1)
        idx, cnt = csa.pool_topk(qI_deq, np.asarray(w)[None], kI_deq, pl,
                                 np.array([int(np.sum(pl >= 0))]), np.array([t]), m, k)
    else:
        raise ValueError(mode)
    sel = idx[0, :cnt[0]].astype(np.int64)
    kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                                  main["B_b"], m, True, sel, d_rope, theta, eps)
    kv_sel_st = round_out(kv_sel, kv_dtype)
    rows = np.concatenate([kv_sel_st, np.asarray(main["C_a"][csa.window_rows(t, n_w)], dtype=np.float64)], axis=0)
    o, lse = csa.attend(np.asarray(q), rows, sink, scale)
    if inv_rope:
        o = csa.inverse_rope(o, t, d_rope, theta)
    new_entry = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                                     main["B_b"], m, True, [E - 1], d_rope, theta, eps)[0]
    return dict(kI=kI, kI_deq=kI_deq, qI_deq=qI_deq, scores=scores[0], idx=idx[0], cnt=int(cnt[0]),
                kv_sel=kv_sel, new_entry=new_entry, new_kI=kI[E - 1],
                out=round_out(o, kv_dtype), out_f64=o, lse=lse)


def hca_decode_seq(main, q, sink, *, L, m, d_rope, theta, eps, n_w, scale, kv_dtype,
                   entries_needed=None, inv_rope=False):
    """One HCA decode step of one sequence: compress the completed block, attend densely.

    main holds C_a, Z_a, B_a (no previous-block branch in c128a).  The new
    token t = L - 1 completes entry E - 1; every entry 0..E-1 is visible.
    """
    E = L // m
    t = L - 1
    kv = csa.compress_range(main["C_a"], main["Z_a"], main["B_a"], None, None, None, m, False,
                            0, E, d_rope, theta, eps, chunk_rows=1 << 16)
    kv_st = round_out(kv, kv_dtype)
    rows = np.concatenate([kv_st, np.asarray(main["C_a"][csa.window_rows(t, n_w)], dtype=np.float64)], axis=0)
    o, lse = csa.attend(np.asarray(q), rows, sink, scale)
    if inv_rope:
        o = csa.inverse_rope(o, t, d_rope, theta)
    return dict(kv=kv, kv_stored=kv_st, new_entry=kv[E - 1], out=round_out(o, kv_dtype),
                out_f64=o, lse=lse)


def csa_decode_at(main, index, q, q_I, w, sink, *, t, m, d_rope, theta, eps, k, n_w, scale,
                  kv_dtype, idx_dtype, inv_rope=False):
    """One CSA decode step of a sequence whose newest token sits at any position t.

    Variable-length batched decode ("DeepSeek-V4技术报告解读", section 3.2, the
    heterogeneous KV cache: compressed blocks plus a per-request state of the
    window and the not yet compressed tail) serves sequences at any t.  Token t
    completes entry (t+1)/m - 1 when (t+1) % m == 0; in any case the query sees
    the E(t) = floor((t+1)/m) entries whose blocks have ended, and the window
    max(0, t-n_w+1)..t.  Rows after t are never read.  q [H][d]; q_I [H_I][d_I];
    w [H_I].
    """
    Et = (t + 1) // m
    qI_deq, _ = quantize_rows(np.asarray(q_I)[None], idx_dtype)
    if Et > 0:
        kI = csa.compress_range(index["C_a"], index["Z_a"], index["B_a"], index["C_b"],
                                index["Z_b"], index["B_b"], m, True, 0, Et, d_rope, theta, eps,
                                chunk_rows=1 << 16)
        kI_deq, _ = quantize_rows(kI, idx_dtype)
        scores = csa.index_scores(qI_deq, np.asarray(w)[None], kI_deq, np.array([t]), m, "bf16")
        idx, cnt = csa.topk(scores, np.array([t]), m, k)
    else:
        kI = np.zeros((0, np.asarray(q_I).shape[-1]))
        scores = np.zeros((1, 0))
        idx, cnt = np.full((1, k), -1, dtype=np.int32), np.zeros(1, dtype=np.int32)
    sel = idx[0, :cnt[0]].astype(np.int64)
    kv_sel = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"], main["Z_b"],
                                  main["B_b"], m, True, sel, d_rope, theta, eps)
    rows = np.concatenate([round_out(kv_sel, kv_dtype).reshape(-1, np.asarray(q).shape[-1]),
                           np.asarray(main["C_a"][csa.window_rows(t, n_w)], dtype=np.float64)], axis=0)
    o, lse = csa.attend(np.asarray(q), rows, sink, scale)
    if inv_rope:
        o = csa.inverse_rope(o, t, d_rope, theta)
    completes = (t + 1) % m == 0
    new_entry = None
    if completes:
        new_entry = csa.compress_entries(main["C_a"], main["Z_a"], main["B_a"], main["C_b"],
                                         main["Z_b"], main["B_b"], m, True, [Et - 1], d_rope,
                                         theta, eps)[0]
    return dict(kI=kI, scores=scores[0], idx=idx[0], cnt=int(cnt[0]), new_entry=new_entry,
                out=round_out(o, kv_dtype), out_f64=o, lse=lse)


def hca_decode_at(main, q, sink, *, t, m, d_rope, theta, eps, n_w, scale, kv_dtype,
                  inv_rope=False):
    """One HCA decode step of a sequence whose newest token sits at any position t: dense
    over the E(t) = floor((t+1)/m) completed entries plus the window."""
    Et = (t + 1) // m
    c = np.asarray(q).shape[-1]
    kv = csa.compress_range(main["C_a"], main["Z_a"], main["B_a"], None, None, None, m, False,
                            0, Et, d_rope, theta, eps, chunk_rows=1 << 16) if Et else np.zeros((0, c))
    rows = np.concatenate([round_out(kv, kv_dtype).reshape(-1, c),
                           np.asarray(main["C_a"][csa.window_rows(t, n_w)], dtype=np.float64)], axis=0)
    o, lse = csa.attend(np.asarray(q), rows, sink, scale)
    if inv_rope:
        o = csa.inverse_rope(o, t, d_rope, theta)
    new_entry = kv[Et - 1] if (t + 1) % m == 0 and Et else None
    return dict(kv=kv, new_entry=new_entry, out=round_out(o, kv_dtype), out_f64=o, lse=lse)
