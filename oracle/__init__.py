"""CPU oracle for the VeriCache hot path -- TEST INFRASTRUCTURE ONLY.

This package is the plain, slow, obviously-correct definition of what the
CUDA library computes.  It works in float64 (numpy) on the host and shares no
code with the CUDA path: no kernels, headers, helpers, tables or constants.

Only three callers may import it:
  * the test suite under ``tests/``,
  * ``__graft_entry__.smoke()`` (which checks one small CUDA invocation
    against it),
  * the ``cpu_baseline`` / ``--impl reference`` leg of ``bench.py``.
The product path never calls it and has no CPU fallback.

Sources (the pages this oracle is written from):
  [P1] "VeriCache: making lossy KV compression exact" (devshah.ca),
       sections "The Tradeoff VeriCache Is Trying to Escape", "The Core Idea",
       "Verifying Without Giving Back the Speedup".
  [P2] "VeriCache: Turning Lossy KV Cache into Lossless LLM Inference"
       (menfem.com knowledge base), sections "Key Contributions",
       "Methodology", "Results", "Limitations".
  [P3] "KV-Cache Compression" (menfem.com knowledge base), section
       "Compression is speculation (VeriCache)".

Modules:
  quant      reference quantiser / dequantiser and code packing
  attention  fp64 softmax attention: quantised draft, token-dropped draft,
             causal block verification
  accept     greedy acceptance (argmax, first mismatch, correction)
  rounds     a toy greedy "model" and the VeriCache round loop, used to pin
             the claim that the emitted stream equals full-cache greedy decoding

Every function states which passage it follows.  Where the pages are silent
the docstring says so and names the reading taken.
"""

from . import quant, attention, accept, rounds  # noqa: F401
