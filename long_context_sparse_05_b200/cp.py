"""Context-parallel CSA decode: each sequence's compressed entries sharded over ranks.

Rank r of G holds a contiguous shard of every sequence's latent cache and index-key
cache (equal shards of a multiple of 256 entries, the indexer's stage; the last rank
takes the rest), and every rank holds the raw rows (window, the block the new token
completes) and the queries.  A step:

  1. local: the last rank, which holds entry E - 1, compresses it into its shard; every
     rank quantises the index queries, scores its shard and keeps its top-k (positions
     shifted by -m * (first entry of the shard), so the causal range is the shard's part
     of the visible entries), and
     turns that top-k into (score, global entry) candidates;
  2. all-gather of the candidates (G x b x k pairs);
  3. merge: the top-k of the gathered candidates, which is exactly the top-k of the whole
     cache (see csa_cp_merge in csa.h); each rank packs the selected rows it holds into
     their slots;
  4. all-reduce (sum) of the packed rows: every rank now has the k selected rows;
  5. attention over those rows and the window, on every rank.

The collectives belong to a communicator, ``DistComm`` (torch.distributed, one process
per GPU); the phases are separate methods, so that several shards can also be driven
phase by phase in one process.  Every compute step is a call of the C ABI.
"""

import math

import torch

from . import _lib as L
from . import runner
from .workloads import Workload

SHARD_ALIGN = 256   # entries: one indexer stage


def shard_bounds(E, world):
    """(first entry, entries) of each rank: equal shards of a multiple of 256 entries, the
    last rank taking the rest (which must not be empty)."""
    S0 = max(SHARD_ALIGN, round(E / world / SHARD_ALIGN) * SHARD_ALIGN)
    if (world - 1) * S0 >= E:
        raise ValueError("too many ranks for E = %d entries (shards of %d)" % (E, S0))
    return [(r * S0, S0 if r < world - 1 else E - (world - 1) * S0) for r in range(world)]


class CPShard:
    """One rank's part of a context-parallel decode batch of workload ``w`` (CSA, FP8 or
    NVFP4 index keys).  ``full`` is a runner.DecodeState of the same inputs with its
    caches built (entries 0 .. E - 2); the shard copies its entries out of it (set-up)."""

    def __init__(self, w: Workload, inputs, rank, world, full, device="cuda"):
        if w.kind != "csa_decode" or w.idx_dtype not in ("fp8", "nvfp4"):
            raise ValueError("context-parallel decode covers CSA decode with FP8 / NVFP4 index keys")
        self.w, self.x, self.rank, self.world, self.device = w, inputs, rank, world, device
        E = w.E
        self.e0, self.n_local = shard_bounds(E, world)[rank]
        S = math.ceil(self.n_local / SHARD_ALIGN) * SHARD_ALIGN   # entries per sequence held
        self.S = S
        self.owner = rank == world - 1          # holds the entry the new token completes
        b, c, k = w.b, w.c, w.k
        dt = runner._TDT[w.dtype]
        hi = self.e0 + self.n_local
        self.kv = torch.zeros((b, S, c), dtype=dt, device=device)
        self.kv[:, :self.n_local] = full.kv_cache[:, self.e0:hi]
        self.kI, self.kIs = runner.alloc_index_cache(b, S, w.c_I, w.idx_dtype, device)
        self.kI.zero_()
        self.kIs.zero_()
        self.kI[:, :self.n_local] = full.kI_cache[:, self.e0:hi]
        if w.idx_dtype == "fp8":
            self.kIs[:, :self.n_local] = full.kI_scales[:, self.e0:hi]
        else:   # NVFP4 scales are tiled per 128 entries: copy whole tiles
            nt = (self.n_local + 127) // 128 * 128
            self.kIs[:, :nt] = full.kI_scales[:, self.e0:self.e0 + nt]
        t = w.n - 1
        self.qpos = torch.full((b, 1), t, dtype=torch.int32, device=device)
        self.qpos_local = torch.full((b, 1), t - w.m * self.e0, dtype=torch.int32, device=device)
        rb = runner.row_bytes(w.idx_dtype, w.c_I)
        self.q_codes = torch.empty((b * w.H_I, rb), dtype=torch.uint8, device=device)
        self.q_scales = (torch.empty((b * w.H_I,), dtype=torch.float32, device=device)
                         if w.idx_dtype == "fp8" else
                         torch.empty((b * w.H_I, w.c_I // 16), dtype=torch.uint8, device=device))
        self.scores = torch.empty((b, 1, self.n_local), dtype=torch.bfloat16, device=device)
        self.idx_l = torch.empty((b, 1, k), dtype=torch.int32, device=device)
        self.cnt_l = torch.empty((b, 1), dtype=torch.int32, device=device)
        self.tk_bytes = L.csa_topk_workspace_size(L.CSA_BF16, b, 1, self.n_local, k)
        self.tk_ws = torch.empty((max(self.tk_bytes, 256),), dtype=torch.uint8, device=device)
        self.cand_s = torch.empty((b, k), dtype=torch.bfloat16, device=device)
        self.cand_i = torch.empty((b, k), dtype=torch.int32, device=device)
        self.gath_s = torch.empty((world, b, k), dtype=torch.bfloat16, device=device)
        self.gath_i = torch.empty((world, b, k), dtype=torch.int32, device=device)
        self.idx = torch.empty((b, k), dtype=torch.int32, device=device)
        self.count = torch.empty((b,), dtype=torch.int32, device=device)
        self.rows_idx = torch.empty((b, 1, k), dtype=torch.int32, device=device)
        self.mg_bytes = L.csa_cp_merge_workspace_size(world, b, k)
        self.mg_ws = torch.empty((self.mg_bytes,), dtype=torch.uint8, device=device)
        self.rows = torch.empty((b, k, c), dtype=dt, device=device)
        self.ap = L.AttnParams(H=w.H, d=c, n_w=w.n_w, scale=w.scale, m=w.m, k=k, dtype=L.DTYPE[w.dtype],
                               d_rope_out=w.d_rope if w.inv_rope else 0, rope_theta=w.theta)
        self.at_bytes = L.csa_sparse_attn_workspace_size(self.ap, b, 1, k)
        self.at_ws = torch.full((max(self.at_bytes, 256),), 0xFF, dtype=torch.uint8, device=device)
        self.out = torch.empty((b, 1, w.H, c), dtype=dt, device=device)
        self.lse = torch.empty((b, 1, w.H), dtype=torch.float32, device=device)
        self.ip = L.IndexParams(H_I=w.H_I, d_I=w.c_I, m=w.m, qk_dtype=L.DTYPE[w.idx_dtype],
                                score_dtype=L.CSA_BF16)

    # -- phase 1: this rank's entries ------------------------------------------------
    def _compress_new_entry(self, stream):
        """Entry E - 1 into this shard, at row E - 1 - e0 of each sequence."""
        w, x = self.w, self.x
        E1 = w.E - 1
        pm = runner.compress_params(w, "main")
        pm.out_entry_offset = self.e0
        L.csa_compress(pm, x["C_a"], x["Z_a"], x["B_a"], x["C_b"], x["Z_b"], x["B_b"], w.b, w.n,
                       E1, 1, self.S, self.kv, None, stream)
        pi = runner.compress_params(w, "index")
        pi.out_entry_offset = self.e0
        L.csa_compress(pi, x["CI_a"], x["ZI_a"], x["BI_a"], x["CI_b"], x["ZI_b"], x["BI_b"], w.b,
                       w.n, E1, 1, self.S, self.kI, self.kIs, stream)

    def phase_local(self, stream=None):
        w, x = self.w, self.x
        if self.owner:
            self._compress_new_entry(stream)
        L.csa_quantize(L.DTYPE[w.dtype], L.DTYPE[w.idx_dtype], x["q_I"], w.b * w.H_I, w.c_I,
                       self.q_codes, self.q_scales, stream)
        L.csa_index_scores(self.ip, self.q_codes, self.q_scales, x["w"], self.kI, self.kIs,
                           self.qpos_local, w.b, 1, self.S, self.n_local, self.scores, stream)
        L.csa_topk(self.scores, L.CSA_BF16, self.qpos_local, w.m, w.b, 1, self.n_local, w.k,
                   self.idx_l, self.cnt_l, self.tk_ws, self.tk_bytes, stream)
        L.csa_cp_candidates(self.scores, self.n_local, self.idx_l, self.cnt_l, w.b, w.k, self.e0,
                            self.cand_s, self.cand_i, stream)
        return self.cand_s, self.cand_i

    # -- phase 2: the global selection and the rows this rank holds --------------------
    def phase_merge(self, stream=None):
        """After gath_s / gath_i hold every rank's candidates (rank-major)."""
        w = self.w
        L.csa_cp_merge(self.gath_s, self.gath_i, self.world, w.b, w.k, self.idx, self.count,
                       self.rows_idx, self.mg_ws, self.mg_bytes, stream)
        L.csa_cp_pack_rows(self.kv, self.S, self.n_local, self.e0, w.c, L.DTYPE[w.dtype], self.idx,
                           self.count, w.b, w.k, self.rows, stream)
        return self.rows

    # -- phase 3: attention over the gathered rows and the window ----------------------
    def phase_attend(self, stream=None):
        """After rows holds the sum over the ranks (every selected row)."""
        w, x = self.w, self.x
        L.csa_sparse_attn(self.ap, x["q"], self.rows, w.k, self.rows_idx, self.count.view(w.b, 1),
                          x["C_a"], w.n, self.qpos, x["sink"], w.b, 1, self.out, self.lse,
                          self.at_ws, self.at_bytes, stream)
        return self.out


class DistComm:
    """The collectives of a step over a torch.distributed process group (NCCL on GPUs)."""

    def __init__(self, group=None):
        self.group = group

    def all_gather(self, out, inp):
        torch.distributed.all_gather_into_tensor(out, inp, group=self.group)

    def all_reduce_sum(self, t):
        torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.SUM, group=self.group)


def decode_step(shard: CPShard, comm, stream=None):
    """One context-parallel decode step of this rank (every rank calls it)."""
    cs, ci = shard.phase_local(stream)
    comm.all_gather(shard.gath_s.view(-1), cs.reshape(-1))
    comm.all_gather(shard.gath_i.view(-1), ci.reshape(-1))
    rows = shard.phase_merge(stream)
    comm.all_reduce_sum(rows)
    return shard.phase_attend(stream)
