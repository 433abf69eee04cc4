"""Context-parallel decode (csa_cp_* and long_context_sparse_05_b200.cp): each sequence's
compressed entries sharded over G ranks, the ranks run here one after another on one GPU
(tests/cp_local.py; no kernel waits on another).

Acceptance: the selection is bit-exact, and the output and lse bit-equal, to the same
step run unsharded through the stage calls (csa_quantize, csa_index_scores, csa_topk,
csa_sparse_attn) on a whole cache holding the same entries.  An entry's score does not
depend on where its key sits, the global top-k is the top-k of the shards' top-k, and
the attention then reads the same rows in the same order.  The selection is also checked
against the oracle within the tie band (the end-to-end acceptance of the decode step).

Source: "DeepSeek Technical Reports", section DSA (attention over the k best entries).
"""

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import cp, runner, synth, workloads
from oracle import csa

from cp_local import LocalGroup
from helpers import f64, topk_band_check

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _unsharded(w, inp, full):
    """The whole cache with entry E - 1 written by csa_compress, then the stage calls."""
    x = inp
    E1 = w.E - 1
    L.csa_compress(runner.compress_params(w, "main"), x["C_a"], x["Z_a"], x["B_a"], x["C_b"],
                   x["Z_b"], x["B_b"], w.b, w.n, E1, 1, full.E_cap, full.kv_cache, None)
    L.csa_compress(runner.compress_params(w, "index"), x["CI_a"], x["ZI_a"], x["BI_a"], x["CI_b"],
                   x["ZI_b"], x["BI_b"], w.b, w.n, E1, 1, full.E_cap, full.kI_cache, full.kI_scales)
    rb = runner.row_bytes(w.idx_dtype, w.c_I)
    codes = torch.empty((w.b * w.H_I, rb), dtype=torch.uint8, device=DEV)
    qs = (torch.empty((w.b * w.H_I,), dtype=torch.float32, device=DEV) if w.idx_dtype == "fp8"
          else torch.empty((w.b * w.H_I, w.c_I // 16), dtype=torch.uint8, device=DEV))
    L.csa_quantize(L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], x["q_I"], w.b * w.H_I, w.c_I, codes, qs)
    qpos = torch.full((w.b, 1), w.n - 1, dtype=torch.int32, device=DEV)
    ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                       score_dtype=L.CSA_BF16)
    scores = torch.empty((w.b, 1, w.E), dtype=torch.bfloat16, device=DEV)
    L.csa_index_scores(ip, codes, qs, x["w"], full.kI_cache, full.kI_scales, qpos, w.b, 1,
                       full.E_cap, w.E, scores)
    idx = torch.empty((w.b, 1, w.k), dtype=torch.int32, device=DEV)
    cnt = torch.empty((w.b, 1), dtype=torch.int32, device=DEV)
    tb = L.csa_topk_workspace_size(L.CSA_BF16, w.b, 1, w.E, w.k)
    tws = torch.empty((max(tb, 256),), dtype=torch.uint8, device=DEV)
    L.csa_topk(scores, L.CSA_BF16, qpos, w.m, w.b, 1, w.E, w.k, idx, cnt, tws, tb)
    ap = L.AttnParams(H=w.H, d=w.c, n_w=w.n_w, scale=w.scale, m=w.m, k=w.k, dtype=L.DTYPE[w.dtype],
                      d_rope_out=w.d_rope if w.inv_rope else 0, rope_theta=w.theta)
    ab = L.csa_sparse_attn_workspace_size(ap, w.b, 1, full.E_cap)
    aws = torch.full((max(ab, 256),), 0xFF, dtype=torch.uint8, device=DEV)
    out = torch.empty((w.b, 1, w.H, w.c), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((w.b, 1, w.H), dtype=torch.float32, device=DEV)
    L.csa_sparse_attn(ap, x["q"], full.kv_cache, full.E_cap, idx, cnt, x["C_a"], w.n, qpos,
                      x["sink"], w.b, 1, out, lse, aws, ab)
    return scores, idx, cnt, out, lse


@pytest.mark.parametrize("base,G,n,inv_rope", [
    ("64k_fp8", 2, 4 * 1500, False),      # shards of 768 + 732 entries
    ("64k_fp8", 3, 4 * 1500, True),       # 512 + 512 + 476
    ("1m_nvfp4", 2, 4 * 3000, False),     # NVFP4 keys: 1536 + 1464, tiled scales split at a tile
    ("64k_fp8", 4, 4 * 1100, False),      # 256 + 256 + 256 + 332
])
def test_cp_decode_equals_the_unsharded_step(base, G, n, inv_rope):
    w0 = workloads.CSA_DECODE_64K if base == "64k_fp8" else workloads.CSA_DECODE_1M
    w = workloads.shrink(w0, b=3 if base == "64k_fp8" else 2, n=n, inv_rope=inv_rope)
    inp = synth.make_inputs(w, device=DEV)
    full = runner.DecodeState(w, inp)
    full.build_caches()
    shards = [cp.CPShard(w, inp, r, G, full) for r in range(G)]
    assert sum(s.n_local for s in shards) == w.E
    assert sum(s.owner for s in shards) == 1
    outs = LocalGroup(shards).step()
    scores, idx, cnt, out, lse = _unsharded(w, inp, full)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    for s in shards:
        assert torch.equal(s.count, cnt.view(-1))
        assert torch.equal(s.idx, idx.view(w.b, -1))
        assert torch.equal(s.out, out)
        assert torch.equal(s.lse, lse)
    # the shards' scores are the whole cache's, entry by entry
    got = torch.cat([s.scores for s in shards], dim=2)
    assert torch.equal(got, scores)
    # the entry the token completes, in the owner's shard
    own = next(s for s in shards if s.owner)
    assert torch.equal(own.kv[:, w.E - 1 - own.e0], full.kv_cache[:, w.E - 1])
    # end-to-end acceptance against the oracle's exact scores, one sequence
    g = {k: f64(v[0]) if v.dim() >= 3 else f64(v) for k, v in inp.items()}
    kI = csa.compress_range(g["CI_a"], g["ZI_a"], g["BI_a"], g["CI_b"], g["ZI_b"], g["BI_b"], w.m,
                            True, 0, w.E, w.d_rope_I, w.theta, w.eps)
    from oracle import pipeline
    kd = pipeline.quantize_rows(kI, w.idx_dtype)[0]
    qd = pipeline.quantize_rows(g["q_I"][0][None], w.idx_dtype)[0]
    exact = csa.index_scores(qd, g["w"][0][None], kd, np.array([w.n - 1]), w.m, "f64")[0]
    topk_band_check(shards[0].idx[0].cpu().numpy(), int(shards[0].count[0]), exact, w.E, w.k)


def test_cp_merge_rejects_bad_arguments():
    ws = torch.empty(256, dtype=torch.uint8, device=DEV)
    s = torch.empty((2, 1, 4), dtype=torch.bfloat16, device=DEV)
    i = torch.empty((2, 1, 4), dtype=torch.int32, device=DEV)
    o = torch.empty((1, 4), dtype=torch.int32, device=DEV)
    c = torch.empty((1,), dtype=torch.int32, device=DEV)
    with pytest.raises(L.CsaError, match="INVALID_ARG"):   # workspace too small
        L.csa_cp_merge(s, i, 2, 1, 4, o, c, o, ws, 16)
    with pytest.raises(L.CsaError, match="INVALID_ARG"):   # no ranks
        L.csa_cp_merge(s, i, 0, 1, 4, o, c, o, ws, 256)
