"""Device-side plumbing around the C ABI for the CSA / HCA workloads.

Allocates caches, outputs and workspaces with torch, fills the parameter
structs from a ``Workload`` and calls the library.  No arithmetic of the method
happens here.
"""

import math

import torch

from . import _lib as L
from .workloads import Workload

_TDT = {"f32": torch.float32, "bf16": torch.bfloat16}


def row_bytes(dtype, d):
    return {"f32": 4 * d, "bf16": 2 * d, "fp8": d, "nvfp4": d // 2}[dtype]


def alloc_index_cache(b, E_cap, c_I, idx_dtype, device):
    """Index-key cache (codes) and its scales for the index-path type."""
    if idx_dtype == "f32":
        return torch.empty((b, E_cap, c_I), dtype=torch.float32, device=device), None
    codes = torch.empty((b, E_cap, row_bytes(idx_dtype, c_I)), dtype=torch.uint8, device=device)
    if idx_dtype == "fp8":
        scales = torch.empty((b, E_cap), dtype=torch.float32, device=device)
    else:
        # tiled NVFP4 key-scale layout: whole tiles of 128 entries per sequence
        e_pad = (E_cap + 127) // 128 * 128
        scales = torch.empty((b, e_pad, c_I // 16), dtype=torch.uint8, device=device)
    return codes, scales


def compress_params(w: Workload, branch="main", out_dtype=None, apply_norm=True):
    c = w.c if branch == "main" else w.c_I
    d_r = w.d_rope if branch == "main" else w.d_rope_I
    od = out_dtype if out_dtype is not None else (w.dtype if branch == "main" else w.idx_dtype)
    return L.CompressParams(m=w.m, overlap=1 if w.overlap else 0, c=c, d_rope=d_r,
                            rope_theta=w.theta, eps=w.eps, apply_norm=1 if apply_norm else 0,
                            in_dtype=L.DTYPE[w.dtype], out_dtype=L.DTYPE[od])


def decode_params(w: Workload, E_cap=None):
    hca = w.kind == "hca_decode"
    return L.DecodeParams(b=w.b, L=w.n, m=w.m, c=w.c, H=w.H, c_I=w.c_I, H_I=w.H_I,
                          d_rope=w.d_rope, d_rope_I=w.d_rope_I, rope_theta=w.theta, eps=w.eps,
                          k=max(w.k, 1), n_w=w.n_w, scale=w.scale, kv_dtype=L.DTYPE[w.dtype],
                          idx_dtype=L.DTYPE.get(w.idx_dtype, 0), hca=1 if hca else 0,
                          E_cap=E_cap if E_cap is not None else w.E,
                          inv_rope=1 if w.inv_rope else 0)


def prefill_params(w: Workload):
    return L.PrefillParams(b=w.b, n=w.n, m=w.m, c=w.c, H=w.H, c_I=w.c_I, H_I=w.H_I,
                           d_rope=w.d_rope, d_rope_I=w.d_rope_I, rope_theta=w.theta, eps=w.eps,
                           k=w.k, n_w=w.n_w, scale=w.scale, kv_dtype=L.DTYPE[w.dtype],
                           idx_dtype=L.DTYPE[w.idx_dtype], score_dtype=L.DTYPE[w.score_dtype],
                           inv_rope=1 if w.inv_rope else 0)


class DecodeState:
    """Caches and buffers of one decode workload on the device.

    ``build_caches()`` compresses entries 0..E-2 of every sequence (the state a
    decode step starts from); ``step()`` runs one fused decode step, which
    compresses entry E-1 and attends.
    """

    def __init__(self, w: Workload, inputs, device="cuda"):
        self.w = w
        self.x = inputs
        self.device = device
        self.E = w.E
        # the FP8 tensor-core indexer reads key scales in whole 16-byte runs: rows of a
        # multiple of 4 entries
        self.E_cap = w.E if w.kind == "hca_decode" else (w.E + 3) // 4 * 4
        self.p = decode_params(w, self.E_cap)
        dt = _TDT[w.dtype]
        self.kv_cache = torch.zeros((w.b, self.E_cap, w.c), dtype=dt, device=device)
        self.hca = w.kind == "hca_decode"
        if not self.hca:
            self.kI_cache, self.kI_scales = alloc_index_cache(w.b, self.E_cap, w.c_I, w.idx_dtype,
                                                              device)
            self.idx = torch.empty((w.b, w.k), dtype=torch.int32, device=device)
            self.count = torch.empty((w.b,), dtype=torch.int32, device=device)
        else:
            self.kI_cache = self.kI_scales = self.idx = self.count = None
        self.out = torch.empty((w.b, w.H, w.c), dtype=dt, device=device)
        self.lse = torch.empty((w.b, w.H), dtype=torch.float32, device=device)
        self.ws_bytes = L.csa_decode_workspace_size(self.p)
        # NaN bytes: a kernel that read workspace it had not written would show up
        self.ws = torch.full((max(self.ws_bytes, 256),), 0xFF, dtype=torch.uint8, device=device)

    def build_caches(self, stream=None):
        w, x = self.w, self.x
        E0 = self.E - 1
        if E0 <= 0:
            return
        cp = compress_params(w, "main")
        L.csa_compress(cp, x["C_a"], x["Z_a"], x["B_a"], x.get("C_b"), x.get("Z_b"), x.get("B_b"),
                       w.b, w.n, 0, E0, self.E_cap, self.kv_cache, None, stream)
        if not self.hca:
            ci = compress_params(w, "index")
            L.csa_compress(ci, x["CI_a"], x["ZI_a"], x["BI_a"], x["CI_b"], x["ZI_b"], x["BI_b"],
                           w.b, w.n, 0, E0, self.E_cap, self.kI_cache, self.kI_scales, stream)

    def tensors(self, q=None, q_I=None, w_=None, out=None):
        x = self.x
        d = dict(C_a=x["C_a"], Z_a=x["Z_a"], C_b=x.get("C_b"), Z_b=x.get("Z_b"), B_a=x["B_a"],
                 B_b=x.get("B_b"), kv_cache=self.kv_cache, kv_win=x["C_a"],
                 q=(q if q is not None else x["q"]), sink=x["sink"],
                 out=(out if out is not None else self.out), lse=self.lse)
        if not self.hca:
            d.update(CI_a=x["CI_a"], ZI_a=x["ZI_a"], CI_b=x["CI_b"], ZI_b=x["ZI_b"],
                     BI_a=x["BI_a"], BI_b=x["BI_b"], kI_cache=self.kI_cache,
                     kI_scales=self.kI_scales, q_I=(q_I if q_I is not None else x["q_I"]),
                     w=(w_ if w_ is not None else x["w"]), idx_out=self.idx, count_out=self.count)
        return d

    def step(self, stream=None, **over):
        L.csa_decode(self.p, self.tensors(**over), self.ws, self.ws_bytes, stream)
        return self.out


class PrefillState:
    """Buffers of one CSA prefill workload on the device."""

    def __init__(self, w: Workload, inputs, device="cuda"):
        self.w = w
        self.x = inputs
        E = w.E
        dt = _TDT[w.dtype]
        self.p = prefill_params(w)
        self.kv_cache = torch.empty((w.b, E, w.c), dtype=dt, device=device)
        self.kI_cache, self.kI_scales = alloc_index_cache(w.b, E, w.c_I, w.idx_dtype, device)
        self.out = torch.empty((w.b, w.n, w.H, w.c), dtype=dt, device=device)
        self.lse = torch.empty((w.b, w.n, w.H), dtype=torch.float32, device=device)
        self.idx = torch.empty((w.b, w.n, w.k), dtype=torch.int32, device=device)
        self.count = torch.empty((w.b, w.n), dtype=torch.int32, device=device)
        self.ws_bytes = L.csa_prefill_workspace_size(self.p)
        # NaN bytes: a kernel that read workspace it had not written would show up
        self.ws = torch.full((max(self.ws_bytes, 256),), 0xFF, dtype=torch.uint8, device=device)

    def run(self, stream=None):
        x = self.x
        t = dict(C_a=x["C_a"], Z_a=x["Z_a"], C_b=x["C_b"], Z_b=x["Z_b"], B_a=x["B_a"], B_b=x["B_b"],
                 CI_a=x["CI_a"], ZI_a=x["ZI_a"], CI_b=x["CI_b"], ZI_b=x["ZI_b"], BI_a=x["BI_a"],
                 BI_b=x["BI_b"], kv_win=x["C_a"], q=x["q"], q_I=x["q_I"], w=x["w"],
                 sink=x["sink"], kv_cache=self.kv_cache, kI_cache=self.kI_cache,
                 kI_scales=self.kI_scales, out=self.out, lse=self.lse, idx_out=self.idx,
                 count_out=self.count)
        L.csa_prefill(self.p, t, self.ws, self.ws_bytes, stream)
        return self.out


def decode_bytes_per_step(w: Workload, k_eff=None):
    """Algorithmic HBM bytes of one decode step (all sequences).

    Index keys E x row (+ scale) are streamed once; the k selected latent rows
    and the n_w window rows are gathered once (1 KiB each at c = 512 bf16);
    q is read and out written once; the compressor reads its 2m (or m) raw
    rows of C and Z (and the index branch), writes one entry.
    """
    eb = 2 if w.dtype == "bf16" else 4
    per = 0
    if w.kind != "hca_decode":
        krow = {"fp8": w.c_I + 4, "nvfp4": w.c_I // 2 + w.c_I // 16, "f32": 4 * w.c_I}[w.idx_dtype]
        per += w.E * krow
        per += (k_eff if k_eff is not None else w.k) * w.c * eb
        per += 2 * 2 * w.m * w.c_I * eb + w.H_I * w.c_I * eb + w.H_I * 4
        per += 2 * 2 * w.m * w.c * eb
    else:
        per += w.E * w.c * eb
        per += 2 * w.m * w.c * eb
    per += w.n_w * w.c * eb
    per += 2 * w.H * w.c * eb
    return per * w.b


def prefill_flops(w: Workload):
    """Causal indexer FLOPs and attention FLOPs of one CSA prefill."""
    t = torch.arange(w.n, dtype=torch.float64)
    Et = torch.floor((t + 1) / w.m)
    idx = float(Et.sum()) * w.H_I * w.c_I * 2 * w.b
    rows = torch.minimum(Et, torch.tensor(float(w.k))) + torch.minimum(t + 1, torch.tensor(float(w.n_w)))
    attn = float(rows.sum()) * w.H * w.c * 4 * w.b
    return idx, attn



def decode_launches_per_step(w: Workload):
    """Kernels one csa_decode call launches (reported by the library)."""
    return L.csa_decode_launch_count(decode_params(w))


def prefill_launches(w: Workload):
    return L.csa_prefill_launch_count(prefill_params(w))


def paged_params(w: Workload, max_pages, num_pages, L_max):
    hca = w.kind == "hca_decode"
    return L.PagedParams(b=w.b, m=w.m, c=w.c, H=w.H, c_I=w.c_I, H_I=w.H_I, d_rope=w.d_rope,
                         d_rope_I=w.d_rope_I, rope_theta=w.theta, eps=w.eps, k=max(w.k, 1),
                         n_w=w.n_w, scale=w.scale, kv_dtype=L.DTYPE[w.dtype],
                         idx_dtype=L.DTYPE.get(w.idx_dtype, 0), hca=1 if hca else 0,
                         max_pages=max_pages, num_pages=num_pages, L_max=L_max,
                         inv_rope=1 if w.inv_rope else 0)


class PagedDecodeState:
    """Paged caches and per-sequence state of one decode workload, for csa_decode_paged.

    ``positions[s]`` is the position t of sequence s's new token (default n - 1 for all).
    Set-up (untimed) compresses every entry completed before t into the pages of the
    sequence (consecutive pages per sequence, then the pages are shuffled and the block
    table follows them), fills the rings of the state with the raw rows before t and
    stages the new token's rows as the step's inputs.
    """

    def __init__(self, w: Workload, inputs, positions=None, device="cuda", shuffle_seed=0):
        self.w, self.x, self.device = w, inputs, device
        b, m, PE = w.b, w.m, L.PAGE_ENTRIES
        self.hca = w.kind == "hca_decode"
        pos = [w.n - 1] * b if positions is None else list(positions)
        self.positions = pos
        self.pos = torch.tensor(pos, dtype=torch.int32, device=device)
        E_fin = [(t + 1) // m for t in pos]
        npages = [max(1, (e + PE - 1) // PE) for e in E_fin]
        self.max_pages = max(npages)
        self.num_pages = sum(npages) + 1                      # one spare page
        first = [sum(npages[:s]) for s in range(b)]
        dt = _TDT[w.dtype]
        rows_total = self.num_pages * PE
        self.kv_pages = torch.zeros((rows_total, w.c), dtype=dt, device=device)
        if not self.hca:
            self.kI_pages, self.kI_scales = alloc_index_cache(1, rows_total, w.c_I, w.idx_dtype,
                                                              device)
            self.kI_pages = self.kI_pages[0]
            self.kI_scales = self.kI_scales[0]
        else:
            self.kI_pages = self.kI_scales = None
        # entries completed before each sequence's new token, compressed into its pages
        for s in range(b):
            E0 = pos[s] // m
            if E0 == 0:
                continue
            cap = npages[s] * PE
            sl = slice(first[s] * PE, first[s] * PE + cap)
            xs = {k: (v[s:s + 1] if v.dim() >= 3 else v) for k, v in inputs.items()}
            L.csa_compress(compress_params(w, "main"), xs["C_a"], xs["Z_a"], xs["B_a"],
                           xs.get("C_b"), xs.get("Z_b"), xs.get("B_b"), 1, w.n, 0, E0, cap,
                           self.kv_pages[sl], None)
            if not self.hca:
                sc = self.kI_scales[sl] if w.idx_dtype == "fp8" else self.kI_scales[sl]
                L.csa_compress(compress_params(w, "index"), xs["CI_a"], xs["ZI_a"], xs["BI_a"],
                               xs["CI_b"], xs["ZI_b"], xs["BI_b"], 1, w.n, 0, E0, cap,
                               self.kI_pages[sl], sc)
        # shuffle the physical pages; the block table follows
        g = torch.Generator(device="cpu").manual_seed(shuffle_seed)
        perm = torch.randperm(self.num_pages, generator=g)     # new page of old page i
        inv = torch.empty_like(perm)
        inv[perm] = torch.arange(self.num_pages)
        def shuffle(t):
            v = t.reshape(self.num_pages, -1)
            return v[inv.to(device)].reshape(t.shape).contiguous()
        self.kv_pages = shuffle(self.kv_pages)
        if not self.hca:
            self.kI_pages = shuffle(self.kI_pages)
            self.kI_scales = shuffle(self.kI_scales)
        bt = torch.full((b, self.max_pages), -1, dtype=torch.int32)
        for s in range(b):
            for j in range(npages[s]):
                bt[s, j] = int(perm[first[s] + j])
        self.block_table = bt.to(device)
        # state rings: raw rows of the tokens before t
        R = m if self.hca else 2 * m
        self.ring = R
        def ring_of(name, c):
            r = torch.zeros((b, R, c), dtype=dt, device=device)
            for s in range(b):
                us = [u for u in range(max(0, pos[s] - R + 1), pos[s])]
                if us:
                    ui = torch.tensor(us, device=device)
                    r[s, ui % R] = inputs[name][s, ui]
            return r
        names = ["C_a", "Z_a"] + ([] if self.hca else ["C_b", "Z_b"])
        self.tails = {"tail_" + n: ring_of(n, w.c) for n in names}
        if not self.hca:
            for n in ("CI_a", "ZI_a", "CI_b", "ZI_b"):
                self.tails["tail_" + n] = ring_of(n, w.c_I)
        self.win = torch.zeros((b, w.n_w, w.c), dtype=dt, device=device)
        for s in range(b):
            us = [u for u in range(max(0, pos[s] - w.n_w + 1), pos[s])]
            if us:
                ui = torch.tensor(us, device=device)
                self.win[s, ui % w.n_w] = inputs["C_a"][s, ui]
        # the new token's rows (the step's inputs)
        ti = self.pos.long()
        ar = torch.arange(b, device=device)
        self.new = {"new_" + n: inputs[n][ar, ti].contiguous() for n in names}
        if not self.hca:
            for n in ("CI_a", "ZI_a", "CI_b", "ZI_b"):
                self.new["new_" + n] = inputs[n][ar, ti].contiguous()
        self.new["new_win"] = inputs["C_a"][ar, ti].contiguous()
        self.L_max = max(pos) + 1
        self.p = paged_params(w, self.max_pages, self.num_pages, self.L_max)
        self.out = torch.empty((b, w.H, w.c), dtype=dt, device=device)
        self.lse = torch.empty((b, w.H), dtype=torch.float32, device=device)
        if not self.hca:
            self.idx = torch.empty((b, w.k), dtype=torch.int32, device=device)
            self.count = torch.empty((b,), dtype=torch.int32, device=device)
        else:
            self.idx = self.count = None
        self.ws_bytes = L.csa_decode_paged_workspace_size(self.p)
        # NaN bytes: a kernel that read workspace it had not written would show up
        self.ws = torch.full((max(self.ws_bytes, 256),), 0xFF, dtype=torch.uint8, device=device)

    def tensors(self, q=None, q_I=None, w_=None, new=None):
        x = self.x
        d = dict(kv_pages=self.kv_pages, block_table=self.block_table, win=self.win,
                 pos=self.pos, B_a=x["B_a"], B_b=x.get("B_b"), sink=x["sink"],
                 q=q if q is not None else x["q"], out=self.out, lse=self.lse)
        d.update(self.tails)
        d.update(new if new is not None else self.new)
        if not self.hca:
            d.update(kI_pages=self.kI_pages, kI_scales=self.kI_scales, BI_a=x["BI_a"],
                     BI_b=x["BI_b"], q_I=q_I if q_I is not None else x["q_I"],
                     w=w_ if w_ is not None else x["w"], idx_out=self.idx, count_out=self.count)
        return d

    def step(self, stream=None, **over):
        L.csa_decode_paged(self.p, self.tensors(**over), self.ws, self.ws_bytes, stream)
        return self.out

    def entry_row(self, s, e):
        """Physical row of entry e of sequence s in the pages."""
        PE = L.PAGE_ENTRIES
        return int(self.block_table[s, e // PE]) * PE + e % PE
