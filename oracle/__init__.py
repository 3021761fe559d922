"""CPU oracle for paged single-query decode attention and its block bookkeeping.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this package:
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may import, call or execute it.  The
oracle shares no code with the CUDA library (no kernels, headers, helpers,
tables or constants); the two meet only at the seeded input generators, which
hold none of the method's arithmetic.

Sources.  Three web pages describe the method; they are cited by short name:

* [Taming the Tail] -- "Taming the Tail: How PagedAttention Solves the
  KV-Cache Fragmentation Crisis in Multi-Tenant LLM Serving"
  (architects-blueprint.vercel.app).
* [vLLM PagedAttention FAQ] -- "vLLM PagedAttention: Eliminating KV Cache
  Memory Fragmentation & 4x Throughput" (tinycto.tv).
* [KV-cache chapter] -- the "g12s-kv-cache" chapter on KV-cache management
  (aicomputerinstitute.com).

Modules.

* ``attention``      -- fp64 decode attention over each sequence's de-paged
  K/V (the plain definition the pages say paging leaves unchanged).
* ``fragmentation``  -- block counts, waste and sharing arithmetic of the
  worked examples.
* ``block_model``    -- a reference model of the block manager's semantics
  (free pool, on-demand allocation, reference counts, fork, copy-on-write),
  kept as plain Python lists and dicts.

Every function here is pinned by ``tests/test_oracle_*.py`` to something other
than itself: values the pages print, closed forms, a library routine
(torch's fp64 scaled-dot-product attention) on contiguous inputs, brute force
on tiny inputs, and invariances.  No function is "parity unpinned".
"""
