"""CPU oracle for paged chunk attention — TEST INFRASTRUCTURE ONLY.

A plain, slow, fp64 numpy restatement of what the CUDA path computes, written
from the pages that describe the method and used only to check that path:

  [pt] "Out of the Memory Barrier: A Highly Memory Efficient Training System for
       LLMs with Million-Token Contexts", gist.science/pt/paper/2602.02108
  [es] the same title, gist.science/es/paper/2602.02108
  [it] the same title, gist.science/it/paper/2602.02108

(three summaries of one paper; section numbers below are the summaries' own).

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The product path (``paged_kv_chunk_query_b200``)
never imports it and shares no code with it: no kernels, helpers, constants or
pre/post-processing.  Inputs come from the seeded generator module, which
holds none of the method's arithmetic.

The oracle works on contiguous (unpaged) KV: paging is a storage detail of the
CUDA path and must not change any result.

Modules
  attention  full causal attention and one chunk's forward/backward over an
             explicit key set (dense or page-sparse)
  sparse     page representatives, group query means, Top-K page choice
  recurrent  the chunk-by-chunk loop over a whole sequence
  pool       the page allocator's free-list policy (SplitMix64 + Fisher-Yates)

Every function here is pinned by tests under ``tests/test_oracle_*.py`` to
facts other than itself (closed forms, finite differences, invariants, brute
force, published generator outputs); none is "parity unpinned".
"""
