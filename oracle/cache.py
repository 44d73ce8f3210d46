"""KV-cache writes, plain definition (oracle; test infrastructure only).

Slot addressing ([P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解",
section 3.3, append_token: a new token goes to the end of the current block, or
to a freshly taken block when the current one is full; section 3.2: blocks are
reached only through the block table).  A token at logical position p of a
sequence is stored in slot

    slot = table[p // block_size] * block_size + p % block_size

of the pool viewed as [num_blocks * block_size, num_kv_heads, head_dim].  A
negative slot marks a padding token that is not written.

Copy-on-write ([P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析",
section 2.2: sequences share prefix blocks and a write to a shared block
first copies it) needs a whole-block copy from a source to a destination block
in both the K and the V pool.

All functions work on the stored bits (any dtype) and return new arrays; the
checks built on them are bit-exact.
"""

import numpy as np


def slot_of(table_row, position, block_size):
    """Slot of logical ``position`` of a sequence with block table ``table_row``."""
    p = int(position)
    return int(table_row[p // block_size]) * block_size + p % block_size


def cache_write(k, v, k_cache, v_cache, slot_mapping):
    """Scatter new-token K/V rows into the pools.

    k, v: [T, Hkv, D]; k_cache, v_cache: [num_blocks, block_size, Hkv, D];
    slot_mapping: int [T].  Returns the updated (k_cache, v_cache) copies.
    Tokens are applied in order, so a slot listed twice keeps the later row.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    bs = kc.shape[1]
    for t, slot in enumerate(np.asarray(slot_mapping).tolist()):
        if slot < 0:
            continue
        kc[slot // bs, slot % bs] = k[t]
        vc[slot // bs, slot % bs] = v[t]
    return kc, vc


def copy_blocks(k_cache, v_cache, pairs):
    """Copy whole blocks ``src -> dst`` in both pools, pairs applied in order.

    pairs: int [n, 2] of (src, dst).  Returns updated copies.
    """
    kc = np.array(k_cache, copy=True)
    vc = np.array(v_cache, copy=True)
    for src, dst in np.asarray(pairs, dtype=np.int64).reshape(-1, 2).tolist():
        kc[dst] = kc[src]
        vc[dst] = vc[src]
    return kc, vc


def scatter_history(Khist, Vhist, table_row, k_cache, v_cache):
    """Place a whole logical history [n, Hkv, D] into the pools via its table."""
    bs = k_cache.shape[1]
    n = Khist.shape[0]
    slots = [slot_of(table_row, p, bs) for p in range(n)]
    return cache_write(Khist, Vhist, k_cache, v_cache, slots)
