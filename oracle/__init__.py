"""Plain CPU oracle for the paged KV-cache decode path.

TEST INFRASTRUCTURE ONLY. Nothing in the product (the ``paged_kv_cache_440_b200``
package, its C ABI or its kernels) imports, calls or links this package. Only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline / reference arm of
``bench.py`` may use it.

Every routine is the plainest statement of what the pages define, in float64 (or
in exact bit/byte arithmetic where the operation is a copy or an encoding):

* ``attention``  -- softmax(q K^T * scale) V over the logically contiguous
  sequence gathered through the block table (no split, no online softmax);
  chunked prefill: every new token attends to the positions up to its own.
* ``cache_ops``  -- append of a step's K/V into the slot it maps to, copy of
  whole physical blocks (copy-on-write), both as byte copies.
* ``quant``      -- per-token-head absmax quantization to INT8 and FP8-E5M2 with
  an fp32 scale, and the matching dequantization.
* ``pool``       -- the pages' KV-bytes formula and block arithmetic.
* ``allocator``  -- a reference model of a refcounted block pool.
* ``prefix_cache`` -- a reference model of the prefix cache: cached full-block
  prefixes as a dict, longest-prefix match by brute force, LRU leaf eviction.

Pinned by ``tests/test_oracle_*.py`` against the pages' worked numbers,
closed forms, invariants, brute force and independent library routines.
"""
