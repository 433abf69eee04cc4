"""Plain float64 oracle of the CSA / HCA attention hot path.

TEST INFRASTRUCTURE ONLY (see ``oracle/__init__.py``).  Nothing here is blocked,
fused or reordered beyond what the definitions state; numpy broadcasting over
independent entries / queries / heads is the only vectorisation.

Notation (one sequence unless a ``b`` axis is named):
    n tokens, m compression rate, c channels, E = n // m entries,
    t query position (0-based), E(t) = floor((t + 1) / m) entries visible to t.
"""

import numpy as np

from . import codecs

NEG_INF = -np.inf


# ---------------------------------------------------------------------------
# (1) KV compressor: pool -> RMSNorm -> partial RoPE
# ---------------------------------------------------------------------------

def compress_weights(Z_a, B_a, Z_b, B_b, m, overlap, i):
    """Softmax weights of entry ``i``: array [R][c], R = 2m (overlap) or m.

    "DeepSeek V4 结构速览", section "C4A Compressor": the previous and the
    current block each get their own logits, the two are stacked with a bias
    added, and a softmax runs per channel over the stacked rows.  The printed
    formula of "DeepSeek-V4技术报告解读" (section CSA) indexes both branches
    over one block; it is read as: rows [m(i-1), mi) of the b-branch with
    bias B_b (previous block) stacked above rows [mi, mi+m) of the a-branch
    with bias B_a (current block).  For i = 0 the previous half has logits
    -inf ("第 0 块时上一块...权重置 -inf").  Without overlap (HCA, c128a) only
    the current block's m rows take part.
    """
    u_a = np.asarray(Z_a[m * i:m * i + m], dtype=np.float64) + np.asarray(B_a, dtype=np.float64)
    if overlap:
        if i == 0:
            u_b = np.full_like(u_a, NEG_INF)
        else:
            u_b = np.asarray(Z_b[m * (i - 1):m * i], dtype=np.float64) + np.asarray(B_b, dtype=np.float64)
        u = np.concatenate([u_b, u_a], axis=0)
    else:
        u = u_a
    mx = np.max(u, axis=0)
    e = np.exp(u - mx)
    return e / np.sum(e, axis=0)


def compress_pool(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, entries):
    """Pooled (pre-norm) entries [len(entries)][c]: per channel, sum over rows of weight * content.

    Content rows are stacked in the same order as the logits: previous block
    from C_b (zeros for i = 0), then current block from C_a
    ("内容同样拼接后按权重加和", section "C4A Compressor").
    """
    entries = np.asarray(entries, dtype=np.int64)
    c = C_a.shape[1]
    out = np.empty((len(entries), c), dtype=np.float64)
    for row, i in enumerate(entries):
        wgt = compress_weights(Z_a, B_a, Z_b, B_b, m, overlap, int(i))
        cont_a = np.asarray(C_a[m * i:m * i + m], dtype=np.float64)
        if overlap:
            if i == 0:
                cont_b = np.zeros_like(cont_a)
            else:
                cont_b = np.asarray(C_b[m * (i - 1):m * i], dtype=np.float64)
            cont = np.concatenate([cont_b, cont_a], axis=0)
        else:
            cont = cont_a
        out[row] = np.sum(wgt * cont, axis=0)
    return out


def compress_pool_vec(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, i0, count):
    """Same arithmetic as ``compress_pool`` for the contiguous entries [i0, i0+count), vectorised.

    Used where the oracle needs tens of thousands of entries (decode caches).
    Tested equal to ``compress_pool`` in the pins.
    """
    c = C_a.shape[1]
    sl = slice(m * i0, m * (i0 + count))
    u_a = np.asarray(Z_a[sl], dtype=np.float64).reshape(count, m, c) + np.asarray(B_a, dtype=np.float64)
    k_a = np.asarray(C_a[sl], dtype=np.float64).reshape(count, m, c)
    if overlap:
        u_b = np.full((count, m, c), NEG_INF)
        k_b = np.zeros((count, m, c))
        j0 = max(i0, 1)
        if j0 < i0 + count:
            slb = slice(m * (j0 - 1), m * (i0 + count - 1))
            nb = i0 + count - j0
            u_b[j0 - i0:] = np.asarray(Z_b[slb], dtype=np.float64).reshape(nb, m, c) + np.asarray(B_b, dtype=np.float64)
            k_b[j0 - i0:] = np.asarray(C_b[slb], dtype=np.float64).reshape(nb, m, c)
        u = np.concatenate([u_b, u_a], axis=1)
        k = np.concatenate([k_b, k_a], axis=1)
    else:
        u, k = u_a, k_a
    mx = np.max(u, axis=1, keepdims=True)
    e = np.exp(u - mx)
    w = e / np.sum(e, axis=1, keepdims=True)
    return np.sum(w * k, axis=1)


def rms_norm(x, eps):
    """RMSNorm with unit gain over the last axis: x / sqrt(mean(x^2) + eps).

    "DeepSeek V4 结构速览", section "C4A Compressor" ("最后过 RMSNorm + RoPE").
    """
    x = np.asarray(x, dtype=np.float64)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps)


def rope_partial(x, pos, d_rope, theta):
    """Rotary embedding on the last ``d_rope`` dims of each row, at position ``pos`` (per row).

    Pairs are interleaved, (x[c-d_r+2j], x[c-d_r+2j+1]) for j < d_r/2, each
    rotated by pos * theta^(-2j/d_r).  The angle is formed in float64 and
    float64 sin/cos are used.  "DeepSeek Technical Reports", section CSA
    ("Partial Rotary Positional Embedding"); "DeepSeek V4 结构速览", section
    "C4A Compressor".
    """
    x = np.array(x, dtype=np.float64, copy=True)
    if d_rope == 0:
        return x
    c = x.shape[-1]
    pos = np.asarray(pos, dtype=np.float64).reshape(-1, 1)
    j = np.arange(d_rope // 2, dtype=np.float64)
    freq = theta ** (-2.0 * j / d_rope)
    ang = pos * freq[None, :]
    cs, sn = np.cos(ang), np.sin(ang)
    x0 = x[:, c - d_rope::2].copy()
    x1 = x[:, c - d_rope + 1::2].copy()
    x[:, c - d_rope::2] = x0 * cs - x1 * sn
    x[:, c - d_rope + 1::2] = x0 * sn + x1 * cs
    return x


def compress_entries(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, entries, d_rope, theta, eps,
                     apply_norm=True):
    """Finished compressed entries: pool, then RMSNorm, then RoPE anchored at p = m * i.

    The RoPE anchor is printed blank on the page; it is read as the first
    token of the current block (p = m * i) for both c4a and c128a.
    """
    entries = np.asarray(entries, dtype=np.int64)
    x = compress_pool(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, entries)
    if apply_norm:
        x = rms_norm(x, eps)
    return rope_partial(x, m * entries, d_rope, theta)


def compress_range(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, i0, count, d_rope, theta, eps,
                   apply_norm=True, chunk_rows=1 << 20):
    """``compress_entries`` for contiguous entries via ``compress_pool_vec``.

    Entries are independent, so they are processed in chunks of about
    ``chunk_rows`` raw rows only to bound host memory.
    """
    c = C_a.shape[1]
    out = np.empty((count, c), dtype=np.float64)
    step = max(1, chunk_rows // m)
    for j0 in range(i0, i0 + count, step):
        nj = min(step, i0 + count - j0)
        x = compress_pool_vec(C_a, Z_a, B_a, C_b, Z_b, B_b, m, overlap, j0, nj)
        if apply_norm:
            x = rms_norm(x, eps)
        out[j0 - i0:j0 - i0 + nj] = rope_partial(x, m * np.arange(j0, j0 + nj), d_rope, theta)
    return out


# ---------------------------------------------------------------------------
# (2) Lightning indexer
# ---------------------------------------------------------------------------

def visible_entries(t, m):
    """E(t) = floor((t+1)/m): entry s is visible to query t iff its block ends at or before t.

    "DeepSeek V4 结构速览", section "Lightning Indexer" (the causal range is
    printed blank); read as: block s ends at m(s+1)-1 <= t.  "DeepSeek
    Technical Reports", section DSA, writes s < q, read as s < t.
    """
    return (np.asarray(t, dtype=np.int64) + 1) // m


def index_scores(q_I, w, k_I, q_pos, m, out_dtype="bf16"):
    """I[t,s] = sum_j w[t,j] * ReLU(q_I[t,j] . k_I[s]), masked to -inf for s >= E(t).

    "DeepSeek Technical Reports", section DSA (lightning-indexer formula);
    "DeepSeek V4 结构速览", section "Lightning Indexer" (ReLU, per-head
    weighted sum, scores kept in BF16).  Inputs are already dequantised
    float64: q_I [T][H_I][d_I], w [T][H_I], k_I [E][d_I].  The exact float64
    score is rounded once to the output type ("bf16" or "f32").
    """
    q_I = np.asarray(q_I, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k_I = np.asarray(k_I, dtype=np.float64)
    dots = np.einsum("tjd,sd->tjs", q_I, k_I)
    sc = np.einsum("tj,tjs->ts", w, np.maximum(dots, 0.0))
    s = np.arange(k_I.shape[0])
    vis = s[None, :] < visible_entries(q_pos, m)[:, None]
    sc = np.where(vis, sc, NEG_INF)
    if out_dtype == "bf16":
        return codecs.round_to_bf16(sc)
    if out_dtype == "f32":
        return sc.astype(np.float32).astype(np.float64)
    return sc


# ---------------------------------------------------------------------------
# (3) Causal top-k
# ---------------------------------------------------------------------------

def topk(scores, q_pos, m, k):
    """Per query: the k highest scores among entries s < E(t), ties to the lower s.

    "DeepSeek Technical Reports", section DSA (Top-k over I[t,:]);
    "DeepSeek V4 结构速览", sections "核心设计" and "Lightning Indexer"
    (k = 512, 1024 for Pro; causal range).  If E(t) <= k every visible entry
    is kept.  Output: idx [T][k] int32 ascending by s, padded with -1, and
    count [T] int32.
    """
    scores = np.asarray(scores, dtype=np.float64)
    T = scores.shape[0]
    idx = np.full((T, k), -1, dtype=np.int32)
    cnt = np.zeros(T, dtype=np.int32)
    for r in range(T):
        ev = int(visible_entries(q_pos[r], m))
        ev = min(ev, scores.shape[1])
        s = np.arange(ev)
        order = np.lexsort((s, -scores[r, :ev]))   # primary: score desc; secondary: s asc
        keep = np.sort(order[:min(k, ev)])
        idx[r, :len(keep)] = keep
        cnt[r] = len(keep)
    return idx, cnt


def pool_topk(q_I, w, k_I, pool, pool_cnt, q_pos, m, k, out_dtype="bf16"):
    """Hierarchical sparse indexer: re-score only a candidate pool, keep the k best of it.

    "DeepSeek Technical Reports", section CSA2 (Hierarchical Sparse Indexer): a
    full indexer scans the whole context for a larger candidate pool; a later
    Reindex layer scores again with its own query, but searches that pool only.
    For query r: the candidates are pool[r, :pool_cnt[r]] that are visible to
    its position (s < E(t)); each is scored exactly as ``index_scores`` scores it
    (rounded once to ``out_dtype``); the k highest are kept, equal scores going to
    the lower entry, and returned ascending by entry, -1 padded, with a count.
    q_I [T][H_I][d_I], w [T][H_I], k_I [E][d_I] (dequantised float64), pool
    [T][P] int entry ids, pool_cnt [T].
    """
    q_I = np.asarray(q_I, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    k_I = np.asarray(k_I, dtype=np.float64)
    T = q_I.shape[0]
    idx = np.full((T, k), -1, dtype=np.int32)
    cnt = np.zeros(T, dtype=np.int32)
    for r in range(T):
        ev = int(visible_entries(q_pos[r], m))
        cand = np.asarray(pool[r, :int(pool_cnt[r])], dtype=np.int64)
        cand = cand[(cand >= 0) & (cand < min(ev, k_I.shape[0]))]
        if len(cand) == 0:
            continue
        dots = k_I[cand] @ q_I[r].T                          # [P][H_I]
        sc = np.maximum(dots, 0.0) @ w[r]                    # [P]
        if out_dtype == "bf16":
            sc = codecs.round_to_bf16(sc)
        elif out_dtype == "f32":
            sc = sc.astype(np.float32).astype(np.float64)
        order = np.lexsort((cand, -sc))                      # score desc, entry asc
        keep = np.sort(cand[order[:min(k, len(cand))]])
        idx[r, :len(keep)] = keep
        cnt[r] = len(keep)
    return idx, cnt


# ---------------------------------------------------------------------------
# (4) Shared-latent MQA with sliding window and sink
# ---------------------------------------------------------------------------

def attend(q, rows, sink, scale):
    """One query over a set of K=V rows: o_h = sum_j e^{l_j} kv_j / (e^{sink_h} + sum_j e^{l_j}).

    l_j = scale * q_h . kv_j.  The sink is a per-head logit in the denominator
    with no value row ("DeepSeek V4 结构速览", section "HCA（c128a 路线）",
    "含 attention sink"); one latent row serves as key and value for all heads
    ("DeepSeek-V4 技术解读", section 2.1, "共享 KV-MQA").  q [H][d],
    rows [R][d], sink [H].  Returns (o [H][d], lse [H]) with
    lse = log(e^{sink} + sum_j e^{l_j}).
    """
    q = np.asarray(q, dtype=np.float64)
    rows = np.asarray(rows, dtype=np.float64)
    sink = np.asarray(sink, dtype=np.float64)
    if rows.shape[0] == 0:
        return np.zeros_like(q), sink.copy()
    lg = scale * (q @ rows.T)                       # [H][R]
    mx = np.maximum(np.max(lg, axis=1), sink)
    e = np.exp(lg - mx[:, None])
    es = np.exp(sink - mx)
    den = es + np.sum(e, axis=1)
    o = (e @ rows) / den[:, None]
    return o, mx + np.log(den)


def window_rows(t, n_w):
    """Raw-token window of query t: positions max(0, t-n_w+1) .. t inclusive.

    "DeepSeek V4 结构速览", section "核心设计" item 3 (a 128-token window on
    uncompressed tokens); the window is concatenated with the selected entries
    without de-duplication (section "CSA（c4a 路线）", "拼接").
    """
    return np.arange(max(0, t - n_w + 1), t + 1)


def inverse_rope(o, t, d_rope, theta):
    """Inverse RoPE on the last ``d_rope`` dims of every head's output, at query position t.

    "DeepSeek V4 结构速览", section "CSA（c4a 路线）" (the last 64 output dims get
    an inverse RoPE) and section "HCA（c128a 路线）" (the same there).  Read as
    the rotation ``rope_partial`` applies at position t, undone: the pairs are
    rotated by -t * theta^(-2j/d_rope).  The values (= keys) carry RoPE at their
    entries' anchors p_s, so the output's rotary part becomes sum_s a_s R(p_s - t) v_s,
    relative to the query.  o [H][d].
    """
    o = np.asarray(o, dtype=np.float64)
    return rope_partial(o, np.full(o.shape[0], -float(t)), d_rope, theta)


def grouped_out_proj(o, W):
    """Grouped output projection: the H heads' outputs in g groups, each projected alone.

    "DeepSeek-V4 技术解读", section 2.1 (分组输出投影: the output is split into g
    groups that are projected separately, cutting the projection's cost g-fold).
    Read as: o [T][H][d] -> group i = heads [i H/g, (i+1) H/g) concatenated
    (H/g * d values); y[t, i] = W[i] @ group_i; the g results are concatenated.
    W [g][d_g][H/g * d].  Returns y [T][g * d_g] in float64.
    """
    o = np.asarray(o, dtype=np.float64)
    W = np.asarray(W, dtype=np.float64)
    T, H, d = o.shape
    g, d_g, K = W.shape
    assert H % g == 0 and K == (H // g) * d
    grouped = o.reshape(T, g, K)
    y = np.einsum("tgk,gnk->tgn", grouped, W)
    return y.reshape(T, g * d_g)


def sparse_attn(q, kv_comp, idx, cnt, kv_win, q_pos, sink, n_w, scale, m=None, inv_rope=None):
    """CSA attention for T queries of one sequence.

    q [T][H][d]; kv_comp [E][d]; idx [T][k] / cnt [T] from ``topk`` (idx None
    means dense over all E(t) visible entries, the HCA case, which needs m);
    kv_win [n][d] raw rows.  ``inv_rope`` = (d_rope, theta) applies ``inverse_rope``
    to each query's output at its position.  Returns (o [T][H][d], lse [T][H]) in
    float64.
    """
    q = np.asarray(q, dtype=np.float64)
    kv_comp = np.asarray(kv_comp, dtype=np.float64)
    T = q.shape[0]
    o = np.zeros_like(q)
    lse = np.zeros(q.shape[:2])
    for r in range(T):
        t = int(q_pos[r])
        if idx is None:
            sel = np.arange(int(visible_entries(t, m)))
        else:
            sel = np.asarray(idx[r, :int(cnt[r])], dtype=np.int64)
        rows = np.concatenate([kv_comp[sel],
                               np.asarray(kv_win[window_rows(t, n_w)], dtype=np.float64)], axis=0)
        o[r], lse[r] = attend(q[r], rows, sink, scale)
        if inv_rope is not None:
            o[r] = inverse_rope(o[r], t, inv_rope[0], inv_rope[1])
    return o, lse


def dense_attn(q, kv_comp, kv_win, q_pos, sink, n_w, scale, m):
    """HCA: attention over every visible compressed entry plus the window.

    "DeepSeek V4 结构速览", sections "核心设计" item 2 and "HCA（c128a 路线）":
    no indexer; dense over all (at most 8192) entries, equivalent to
    top-k = 8192.
    """
    return sparse_attn(q, kv_comp, None, None, kv_win, q_pos, sink, n_w, scale, m=m)
