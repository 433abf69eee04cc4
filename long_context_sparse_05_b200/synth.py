"""Seeded synthetic inputs for the CSA / HCA workloads.

This module only draws random numbers; it holds none of the method's
arithmetic, and both the CUDA path and the CPU oracle consume exactly the
tensors it returns.

Recipe: every tensor has a fixed id (``TENSOR_ID``) and is drawn from its own
torch generator seeded with ``seed * 1_000_003 + id``: float32 normals (or
uniforms) times the stated spread, then cast to the workload's storage type
(round to nearest even).  Distributions:

* raw latents C, compression logits Z, query heads q, index queries q_I and
  the per-head sink logit: N(0, 1);
* positional biases B (always float32, [m][c]): N(0, 0.5^2), i.e. std 0.5;
* indexer head weights w (float32): U(0, 1) / w_div (4 tiny, 64 otherwise).

Tensors live on ``device``; the same seed gives different values on CPU and
CUDA (different generators), so a test always takes both sides' inputs from
one draw.
"""

import torch

TENSOR_ID = {
    "C_a": 0, "Z_a": 1, "C_b": 2, "Z_b": 3, "B_a": 4, "B_b": 5,
    "CI_a": 6, "ZI_a": 7, "CI_b": 8, "ZI_b": 9, "BI_a": 10, "BI_b": 11,
    "q": 12, "q_I": 13, "w": 14, "sink": 15, "W_o": 16,
}

_TORCH_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def draw(name, shape, seed, device="cpu", dtype="f32", dist="normal", spread=1.0):
    g = torch.Generator(device=device)
    g.manual_seed(seed * 1_000_003 + TENSOR_ID[name])
    if dist == "normal":
        x = torch.randn(shape, generator=g, device=device, dtype=torch.float32)
    else:
        x = torch.rand(shape, generator=g, device=device, dtype=torch.float32)
    if spread != 1.0:
        x.mul_(spread)
    return x.to(_TORCH_DT[dtype])


def make_inputs(w, device="cpu", T=None, b=None):
    """All inputs of workload ``w`` as a dict of torch tensors on ``device``.

    Shapes (batch outermost, row-major):
      C_a, Z_a, C_b, Z_b   [b][n][c]      (C_b / Z_b absent for HCA)
      B_a, B_b             [m][c]  float32
      CI_*, ZI_*           [b][n][c_I],  BI_* [m][c_I]   (CSA only)
      q                    [b][T][H][c]
      q_I                  [b][T][H_I][c_I]  (CSA only)
      w                    [b][T][H_I]  float32          (CSA only)
      sink                 [H]  float32
    T is n for prefill and 1 for decode (the token t = n - 1).
    """
    b = w.b if b is None else b
    T = w.T if T is None else T
    dt = w.dtype
    d = {}
    d["C_a"] = draw("C_a", (b, w.n, w.c), w.seed, device, dt)
    d["Z_a"] = draw("Z_a", (b, w.n, w.c), w.seed, device, dt)
    d["B_a"] = draw("B_a", (w.m, w.c), w.seed, device, "f32", spread=0.5)
    if w.overlap:
        d["C_b"] = draw("C_b", (b, w.n, w.c), w.seed, device, dt)
        d["Z_b"] = draw("Z_b", (b, w.n, w.c), w.seed, device, dt)
        d["B_b"] = draw("B_b", (w.m, w.c), w.seed, device, "f32", spread=0.5)
    if w.c_I:
        d["CI_a"] = draw("CI_a", (b, w.n, w.c_I), w.seed, device, dt)
        d["ZI_a"] = draw("ZI_a", (b, w.n, w.c_I), w.seed, device, dt)
        d["CI_b"] = draw("CI_b", (b, w.n, w.c_I), w.seed, device, dt)
        d["ZI_b"] = draw("ZI_b", (b, w.n, w.c_I), w.seed, device, dt)
        d["BI_a"] = draw("BI_a", (w.m, w.c_I), w.seed, device, "f32", spread=0.5)
        d["BI_b"] = draw("BI_b", (w.m, w.c_I), w.seed, device, "f32", spread=0.5)
        d["q_I"] = draw("q_I", (b, T, w.H_I, w.c_I), w.seed, device, dt)
        d["w"] = draw("w", (b, T, w.H_I), w.seed, device, "f32", dist="uniform",
                      spread=1.0 / w.w_div)
    d["q"] = draw("q", (b, T, w.H, w.c), w.seed, device, dt)
    d["sink"] = draw("sink", (w.H,), w.seed, device, "f32")
    return d
