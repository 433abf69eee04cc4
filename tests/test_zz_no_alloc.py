"""The allocation-free attention entry point (csa_sparse_attn_noalloc).

Some callers cannot allocate device memory (a plugin inside a host framework
that owns all device memory, or a latency-critical loop that must never call
cudaMalloc).  For them the library keeps the split partials of the attention
kernel in one fixed device array.  This file checks, through the C ABI, that
the entry point gives the same output as csa_sparse_attn with a caller
workspace, on two calls in a row with different problems (so stale scratch
from the first call cannot leak into the second), and that a problem needing
more scratch than the array holds is rejected.  It is collected last so that a
failure here does not hide any other test; it also passes alone in a fresh
process.
"""

import math

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import synth
from oracle import csa

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _case(b, E, n, k, seed, dense):
    H, d, n_w = 64, 512, 128
    rng = np.random.default_rng(seed)
    q = synth.draw("q", (b, 1, H, d), seed, DEV, "bf16")
    kv = synth.draw("C_b", (b, E, d), seed, DEV, "bf16")
    win = synth.draw("C_a", (b, n, d), seed, DEV, "bf16")
    sink = synth.draw("sink", (H,), seed, DEV, "f32")
    m = n // E
    qpos = np.full((b, 1), n - 1, np.int32)
    qpos[-1, 0] = n // 2
    if dense:
        idx = cnt = None
    else:
        idx = np.full((b, 1, k), -1, np.int32)
        cnt = np.zeros((b, 1), np.int32)
        for s in range(b):
            idx[s], cnt[s] = csa.topk(rng.normal(size=(1, E)), qpos[s], m, k)
        idx = torch.from_numpy(idx).to(DEV)
        cnt = torch.from_numpy(cnt).to(DEV)
    p = L.AttnParams(H=H, d=d, n_w=n_w, scale=1.0 / math.sqrt(d), m=m, k=0 if dense else k,
                     dtype=L.CSA_BF16)
    return dict(p=p, q=q, kv=kv, win=win, sink=sink, qpos=torch.from_numpy(qpos).to(DEV),
                idx=idx, cnt=cnt, b=b, E=E, n=n, H=H, d=d)


def _with_workspace(c):
    out = torch.empty((c["b"], 1, c["H"], c["d"]), dtype=torch.bfloat16, device=DEV)
    lse = torch.empty((c["b"], 1, c["H"]), dtype=torch.float32, device=DEV)
    wsb = L.csa_sparse_attn_workspace_size(c["p"], c["b"], 1, c["E"])
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes: no read before write
    L.csa_sparse_attn(c["p"], c["q"], c["kv"], c["E"], c["idx"], c["cnt"], c["win"], c["n"],
                      c["qpos"], c["sink"], c["b"], 1, out, lse, ws, wsb)
    return out, lse, wsb


def _no_alloc(c):
    out = torch.full((c["b"], 1, c["H"], c["d"]), float("nan"), dtype=torch.bfloat16, device=DEV)
    lse = torch.full((c["b"], 1, c["H"]), float("nan"), dtype=torch.float32, device=DEV)
    L.csa_sparse_attn_noalloc(c["p"], c["q"], c["kv"], c["E"], c["idx"], c["cnt"], c["win"], c["n"],
                              c["qpos"], c["sink"], c["b"], 1, out, lse)
    return out, lse


def test_noalloc_matches_workspace_entry_point_twice():
    # dense decode splits each query over more CTAs than a cluster holds, so its split
    # partials go through scratch; two calls in a row with different shapes
    first = _case(b=4, E=1500, n=6000, k=0, seed=71, dense=True)
    second = _case(b=3, E=700, n=2800, k=0, seed=72, dense=True)
    # top-k selection: splits merge inside a cluster, no scratch; the entry points still agree
    third = _case(b=4, E=1500, n=6000, k=512, seed=73, dense=False)
    for c, needs_scratch in ((first, True), (second, True), (third, False)):
        ref, ref_lse, wsb = _with_workspace(c)
        if needs_scratch:
            assert wsb > 0, "this shape must use split scratch, or the test checks nothing"
        assert wsb <= L.NOALLOC_SCRATCH_BYTES
        got, got_lse = _no_alloc(c)
        torch.cuda.synchronize()
        assert torch.isfinite(got.float()).all()
        # the same kernels on the same inputs with the same split plan: bit for bit equal
        assert torch.equal(got, ref), (got.float() - ref.float()).abs().max().item()
        assert torch.equal(got_lse, ref_lse)
        assert L.csa_device_error() == 0


def test_noalloc_rejects_problems_beyond_its_scratch():
    # A dense decode of short sequences whose split partials still exceed the fixed
    # scratch: every query is split over many CTAs, one 128 KB partial each.  The
    # buffers are real and of the right size, so were the size check ever lost the
    # call would run a valid problem and the output check below would fail.
    H, d, n_w, m = 64, 512, 128, 4
    E, n = 256, 1024
    p = L.AttnParams(H=H, d=d, n_w=n_w, scale=1.0 / math.sqrt(d), m=m, k=0, dtype=L.CSA_BF16)
    sizes = {b: L.csa_sparse_attn_workspace_size(p, b, 1, E) for b in range(1, 149)}
    big = [b for b, need in sizes.items() if need > L.NOALLOC_SCRATCH_BYTES]
    assert big, sizes
    b = big[0]
    c = _case(b=b, E=E, n=n, k=0, seed=74, dense=True)
    out = torch.zeros((b, 1, H, d), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(L.CsaError, match="INVALID_ARG"):
        L.csa_sparse_attn_noalloc(c["p"], c["q"], c["kv"], E, None, None, c["win"], n, c["qpos"],
                                  c["sink"], b, 1, out)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out).item() == 0     # nothing was launched
