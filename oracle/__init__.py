"""CPU oracle for the paged decode path: TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline legs of
``bench.py`` may import or run anything in this package. The product path
(``paged_kv_cache_driven_b200``) never does, and the two share no code: the only
thing both sides see is the seeded synthetic inputs.

Contents, each pinned by ``-m "not gpu"`` tests in ``tests/test_oracle_*.py``:

* ``decode``          -- fp64 paged decode attention (C++ in ``oracle.cpp``):
                         softmax(q K^T * scale) V gathered through block tables,
                         and the per-partition (m, l, acc) statistics of a split.
* ``append``          -- the slot_mapping scatter of new tokens' K/V, in numpy.
* ``allocator_model`` -- the block pool: free list, on-demand growth, block
                         tables, slot mappings, waste statistics.
* ``waste``           -- the memory-waste arithmetic of static reservation
                         versus paged allocation.

Every function names the passage of the pages it follows. The pages are:
"PagedAttention" (llm-engineer.pages.dev, LLM inference / vLLM card),
"vLLM KV Cache and PagedAttention Explained" (hrletsgo.me), and
"vLLM의 PagedAttention 아키텍처와 GPU 메모리 최적화 원리" (velog.io, @min_tech).
No function here is "parity unpinned".
"""
