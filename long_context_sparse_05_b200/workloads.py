"""The five CSA / HCA workloads, as plain shape and type descriptions.

No arithmetic of the method lives here.  Sizes follow the configurations the
library is measured on: a tiny fp32 CSA prefill, CSA decode at 64K context
(FP8 indexer), CSA prefill at 32K (FP8 indexer), HCA decode at 1M context and
CSA decode at 1M context (NVFP4 indexer).
"""

from dataclasses import dataclass, replace
import math


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str            # "csa_prefill" | "csa_decode" | "hca_decode"
    b: int               # sequences
    n: int               # tokens per sequence (context length L for decode)
    m: int               # compression rate
    c: int               # latent dim (K = V)
    H: int               # query heads (head dim d = c)
    c_I: int = 0         # index-key dim d_I (0: no indexer)
    H_I: int = 0         # indexer heads
    d_rope: int = 64     # rotary dims at the end of each compressed entry
    d_rope_I: int = 64   # rotary dims at the end of each index key
    theta: float = 10000.0
    eps: float = 1e-6
    k: int = 0           # top-k (0: dense, HCA)
    n_w: int = 128       # raw sliding-window length
    scale: float = 0.0   # attention logit scale
    dtype: str = "bf16"  # storage type of C, Z, q, caches and outputs ("f32" | "bf16")
    idx_dtype: str = "fp8"     # index path: "f32" | "fp8" | "nvfp4"
    score_dtype: str = "bf16"  # indexer score storage ("f32" | "bf16")
    w_div: float = 64.0  # indexer head weights ~ U(0,1) / w_div
    seed: int = 0
    inv_rope: bool = False   # inverse RoPE on the last d_rope output dims

    @property
    def E(self):
        return self.n // self.m

    @property
    def overlap(self):
        return self.m > 1 and self.kind != "hca_decode"

    @property
    def T(self):
        """Queries per sequence."""
        return self.n if self.kind == "csa_prefill" else 1


TINY = Workload("csa_prefill_tiny_f32", "csa_prefill", b=1, n=1024, m=4, c=64, H=4, c_I=32, H_I=4,
                d_rope=16, d_rope_I=16, k=16, n_w=16, scale=1.0 / 8.0, dtype="f32",
                idx_dtype="f32", score_dtype="f32", w_div=4.0, seed=0)

CSA_DECODE_64K = Workload("csa_decode_64k_fp8", "csa_decode", b=16, n=65536, m=4, c=512, H=64,
                          c_I=128, H_I=64, k=512, scale=1.0 / math.sqrt(512), idx_dtype="fp8",
                          seed=2)

CSA_PREFILL_32K = Workload("csa_prefill_32k_fp8", "csa_prefill", b=1, n=32768, m=4, c=512, H=64,
                           c_I=128, H_I=64, k=512, scale=1.0 / math.sqrt(512), idx_dtype="fp8",
                           seed=3)

HCA_DECODE_1M = Workload("hca_decode_1m", "hca_decode", b=8, n=1 << 20, m=128, c=512, H=64,
                         k=0, scale=1.0 / math.sqrt(512), idx_dtype="none", seed=4)

CSA_DECODE_1M = Workload("csa_decode_1m_nvfp4", "csa_decode", b=4, n=1 << 20, m=4, c=512, H=64,
                         c_I=128, H_I=64, k=1024, scale=1.0 / math.sqrt(512), idx_dtype="nvfp4",
                         seed=5)

ALL = {w.name: w for w in (TINY, CSA_DECODE_64K, CSA_PREFILL_32K, HCA_DECODE_1M, CSA_DECODE_1M)}


def shrink(w, **kw):
    """A smaller copy of a workload (same kind, types and dims) for fast parity cases."""
    return replace(w, **kw)
