"""B200-native (sm_100a) Compressed Sparse Attention / Heavily Compressed Attention hot path.

The computation lives in ``libcsa.so`` (C ABI in ``include/csa.h``); this
package is its Python binding (``_lib``), device plumbing (``runner``), the
workload descriptions (``workloads``) and the seeded input generator
(``synth``).  Calling any ``csa_*`` function raises if the library is not
built: there is no CPU fallback.
"""

from ._lib import (CSA_BF16, CSA_F32, CSA_FP8_E4M3, CSA_NVFP4, DTYPE, AttnParams,  # noqa: F401
                   CompressParams, CsaError, DecodeParams, IndexParams, PrefillParams, csa_compress,
                   csa_decode, csa_decode_workspace_size, csa_index_scores, csa_prefill,
                   csa_prefill_workspace_size, csa_quantize, csa_sparse_attn,
                   csa_sparse_attn_workspace_size, csa_status_string, csa_topk, lib)
from . import workloads  # noqa: F401
