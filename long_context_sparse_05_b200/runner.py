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
