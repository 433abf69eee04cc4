"""CPU oracle for the Compressed Sparse Attention (CSA / HCA) hot path.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  The product path (the CUDA library and its Python binding) never
calls it, and it shares no code with that path.

Everything here is a plain, slow, obviously-correct restatement of what the
pages define, in float64 (numpy) unless a step fixes its own precision (the
FP8 / NVFP4 quantisers decide codes in float32, as the format definitions and
the kernels do).  Each function cites the page and section it follows:

* "DeepSeek Technical Reports" (gh-shinku.github.io), section DSA: the
  lightning-indexer formula and the top-k attention formula.
* "DeepSeek-V4技术报告解读" (deepseek.csdn.net), section
  "Compressed Sparse Attention (CSA)": the compressor formula with positional
  bias B (printed garbled; read as described in ``csa.compress_pool``).
* "DeepSeek V4 结构速览" (riverclouds.net), sections "核心设计",
  "CSA（c4a 路线）", "C4A Compressor", "Lightning Indexer",
  "HCA（c128a 路线）": block geometry, the operator graph, per-channel softmax,
  block-0 padding, RMSNorm + RoPE, the FP4 index path, the sink.

Parity status per function is stated in each docstring; functions with no
independent pin say "parity unpinned".
"""

from . import codecs, csa  # noqa: F401
