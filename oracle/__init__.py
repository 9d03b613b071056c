"""fp64 CPU oracle for paged decode attention and its block bookkeeping.

TEST INFRASTRUCTURE, NOT THE PRODUCT. Only ``tests/``, ``__graft_entry__.smoke()``
and ``bench.py`` (its CPU-baseline leg and its ``--impl reference`` arm) may
import anything from this package. The CUDA library under
``paged_kv_cache_319_b200`` never imports it and shares no code with it.

The pages this oracle restates (cited by title and section everywhere in it):

* "Your GPU was mostly empty: how PagedAttention turned KV cache waste into
  2-4x throughput" (blog.teqners.com), abbreviated "Your GPU was mostly empty".
* "vLLM and PagedAttention" (interviewsvector.com).
* "PagedAttention: KV cache memory management" (aitechjournal.org),
  abbreviated "PagedAttention KV cache memory management".

Modules:

* :mod:`oracle.block_manager` - logical-to-physical block bookkeeping:
  allocate on growth, fork with reference counts, block-level copy-on-write,
  release to a shared free pool.
* :mod:`oracle.cache` - the two cache-content operations (scatter of new
  tokens into their slots, whole-block copies for copy-on-write).
* :mod:`oracle.attention` - decode attention over a paged cache: gather each
  sequence's blocks into contiguous K/V, then softmax(q K^T * scale) V in
  fp64; plus the partition / log-sum-exp merge used for long contexts.
* :mod:`oracle.capacity` - the KV bytes-per-token capacity model and the
  waste measures.
* :mod:`oracle.numerics` - decoding of fp16 / bf16 bit patterns to fp64.

Every function is pinned by ``-m "not gpu"`` tests against something other
than itself: the worked numbers the pages print, closed forms, invariants,
a library routine (torch SDPA in fp64) and scalar brute force.
"""
