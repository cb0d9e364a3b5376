"""CPU oracle for paged decode attention — TEST INFRASTRUCTURE, not product code.

A plain, slow, obviously correct restatement of what the paged attention hot
path computes, written from three pages:

  * "Paged Attention" (klaylearn.com glossary)
  * "PagedAttention — AI Glossary" (modelrefs.com)
  * "What is paged attention in vLLM, and why does it matter?" (interview.clozo.ai)

`blocks` covers the block arithmetic and a reference block manager (free list,
reference counts, copy-on-write). `attention` covers the cache writes (append,
block copy, block swap) and decode and causal (chunked) prefill attention in
float64 over the logically contiguous context that the block table describes.
`quant` covers the 8-bit E4M3 cache format (encode with round-to-nearest-even
and saturation, exact decode, per-head scales).

Only the test suite, the smoke check and the benchmark's CPU-baseline leg may
import this package. It shares no code with the CUDA library and the library
never imports it. Every function is pinned by the `-m "not gpu"` tests against
numbers the pages print, closed forms, a library routine or brute force.
"""

from . import attention, blocks  # noqa: F401
