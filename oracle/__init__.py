"""CPU oracle for the paged-KV-cache decode path.

TEST INFRASTRUCTURE ONLY.  Nothing in the product package imports this
package; only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline /
reference leg of ``bench.py`` may import or run it.  It shares no code with the
CUDA path: the two meet only through the seeded input generators in
``paged_kv_cache_381_b200.workloads``, which hold none of the method's
arithmetic.

Every function is a plain, slow, obviously-correct restatement of what the
pages define, in float64 for all floating-point work:

* ``numerics``       -- exact widening of the stored KV dtypes to float64.
* ``attention``      -- single-query scaled-dot-product decode attention over a
                        sequence's KV history, and the same read through a
                        block table over non-contiguous physical blocks.
* ``cache``          -- the slot-mapping scatter of new-token K/V into the
                        block pool, and the whole-block copy used by
                        copy-on-write.
* ``block_manager``  -- free-list / ref-count / block-table bookkeeping.
* ``scheduler``      -- iteration-level admission (FCFS, stop at the first
                        request that does not fit), finish and preemption.

Pages cited (by title) throughout:

[P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解"
     (111cn.net) -- section 2.2 (Continuous Batching scheduler pseudocode),
     section 3.2 (virtual-memory-style paging), section 3.3 (block manager
     code: allocate / append_token).
[P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析" (gtnt.cn) --
     section 2.1 (Block with ref_count, data of shape
     (BLOCK_SIZE, NUM_HEADS, HEAD_SIZE)), section 2.2 (memory pooling,
     copy-on-write, block-level kernel scheduling), section 3.2 (preemptive
     scheduling), section 6.2 (paged_attention_kernel(out, q, k, v,
     block_tables) signature).
[P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置"
     (yunthe.com) -- section "PagedAttention分页注意力机制原理" (block table,
     the kernel resolves physical addresses through it, sharing of prefix
     blocks by reference, free-block pool) and section
     "连续批处理Continuous Batching配置".

Parity status: every function here is pinned by tests/test_oracle_*.py against
something other than itself (brute force, closed forms, a library attention
routine, paging invariants, hand-computed traces); none is "parity unpinned".
"""

from . import numerics, attention, cache, block_manager, scheduler  # noqa: F401
