"""Reference oracle for paged decode attention -- TEST INFRASTRUCTURE ONLY.

This package is a plain, slow, obviously-correct CPU restatement of what the
paged KV cache computes, written in float64 NumPy and pure Python from the
three pages that describe the method:

* "Paged attention in LLMs" (bibekananda.in): fixed-size blocks, the block
  table, the worked example, the waste bound, prefix sharing.
* the zenaique quiz page "PagedAttention (vLLM)": the code sketch
  "Conceptual: PagedAttention block lookup" (gather through the block table,
  then standard scaled-dot-product attention), and the comparison table
  (copy-on-write blocks for beam search).
* "Paged Attention" (mbrenndoerfer.com): motivation only.

Only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import it.  The product path
(the CUDA library and its Python binding) never imports, calls or links it,
and this package imports nothing from the product.

Modules
-------
paged_attention  -- reshape_and_cache, copy_blocks, decode (fp64)
block_allocator  -- free list / refcount / copy-on-write allocator model
accounting       -- slot accounting of the contiguous vs paged layouts

Parity status: every function here is pinned by ``tests/test_oracle_*.py``
against values printed on the pages (``tests/golden/``), closed forms,
invariants and library routines (numpy indexing, torch SDPA in fp64).
No function is "parity unpinned".
"""

from . import accounting, block_allocator, paged_attention  # noqa: F401
