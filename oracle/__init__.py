"""fp64 CPU oracle for the tiled attention forward and its variants.

TEST INFRASTRUCTURE ONLY.  Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package.  It shares no code
with the CUDA library and never imports it; the product path never calls it.

Sources (cited by page title and section throughout):

* [FA-trading]  "Can a full-day context beat one minute? Flash attention and
  the sequence-length question" (marketmaker.cc blog, Thai): sections "Why
  attention is memory-bound", "The Flash Attention algorithm", "Online
  softmax recurrence", "Backward: recompute instead of store", "FA2",
  "Causal masking", "Integration in eight lines", "Correctness check".
* [FA4-overview] "FlashAttention 4: fast, memory-saving attention for LLMs"
  (linux-konsole, Vietnamese): sections "What is new in FlashAttention 4",
  "Software exponent on CUDA cores", "Smarter online softmax rescaling".
* [FP4-FA4]  "Hardware-Aware FP4 FlashAttention-4" (gist.science lay summary,
  Chinese): the Direct-P mapping and the quantise-after-exp baseline.
* [INT-FA]   "INT-FlashAttention: an INT8 quantisation architecture compatible
  with FlashAttention" (hoodcat.net news piece, Spanish): token-level INT8
  Q/K/V with INT8 GEMMs in the forward.

Modules:

* ``oracle.attention`` -- the plain definition (materialised S and P), the
  pages' blockwise algorithm, the lazy-rescale form, split-KV + combine.
* ``oracle.lowp``      -- INT8 and NVFP4 quantisers and step-by-step
  emulations of the quantised forwards.
"""
from . import attention, lowp  # noqa: F401
