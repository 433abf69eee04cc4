"""Output epilogues on the GPU: the grouped output projection (tcgen05 GEMM per head group)
against the oracle.  Inverse RoPE is fused into the attention kernels and checked with
them (test_gpu_stages.py, test_gpu_e2e.py).

Source: "DeepSeek-V4 技术解读", section 2.1 (分组输出投影).  Acceptance: element-wise
|gpu - ref| <= 1e-2 (|ref| + rms(ref)): bf16 inputs, float32 accumulation, one bf16
rounding of the result (at most 2^-8 relative).
"""

import math

import numpy as np
import pytest
import torch

from long_context_sparse_05_b200 import _lib as L
from long_context_sparse_05_b200 import synth
from oracle import csa

from helpers import assert_rel_close, f64

pytestmark = pytest.mark.gpu
DEV = "cuda"


@pytest.mark.parametrize("T,H,d,g,d_g", [
    (16, 64, 512, 8, 1024),     # decode batch: few tokens, the K dimension split
    (300, 64, 512, 8, 1024),    # several token tiles and a ragged tail, no split
    (5, 8, 64, 2, 256),         # small heads: K = 256
    (129, 64, 512, 4, 256),     # four groups of 16 heads (K = 8192)
])
def test_grouped_out_proj(T, H, d, g, d_g):
    K = (H // g) * d
    o = synth.draw("q", (T, H, d), 81, DEV, "bf16")
    W = synth.draw("W_o", (g, d_g, K), 82, DEV, "bf16", spread=1.0 / math.sqrt(K))
    y = torch.full((T, g * d_g), float("nan"), dtype=torch.bfloat16, device=DEV)
    wsb = L.csa_out_proj_workspace_size(T, H, d, g, d_g)
    ws = torch.full((max(wsb, 256),), 0xFF, dtype=torch.uint8, device=DEV)   # NaN bytes
    L.csa_out_proj(o, W, T, H, d, g, d_g, y, ws, wsb)
    torch.cuda.synchronize()
    assert L.csa_device_error() == 0
    if T == 16:
        assert wsb > 0, "the few-token case should split K"
    rows = np.arange(T) if T <= 32 else np.unique(np.concatenate([[0, 1, 127, 128, T - 1],
                                                                  np.random.default_rng(T).integers(0, T, 12)]))
    ref = csa.grouped_out_proj(f64(o[torch.from_numpy(rows).to(DEV)]), f64(W))
    assert_rel_close(f64(y[torch.from_numpy(rows).to(DEV)]), ref, 1e-2, "grouped projection")


def test_grouped_out_proj_rejects_unsupported_shapes():
    o = torch.zeros((4, 64, 512), dtype=torch.bfloat16, device=DEV)
    W = torch.zeros((8, 1000, 4096), dtype=torch.bfloat16, device=DEV)
    y = torch.zeros((4, 8000), dtype=torch.bfloat16, device=DEV)
    with pytest.raises(L.CsaError, match="INVALID_ARG"):
        L.csa_out_proj(o, W, 4, 64, 512, 8, 1000, y)          # d_g not a multiple of 256
    with pytest.raises(L.CsaError, match="INVALID_ARG"):
        L.csa_out_proj(o, W, 4, 64, 512, 7, 1024, y)          # H not a multiple of g
