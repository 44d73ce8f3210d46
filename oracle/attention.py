"""Decode attention, plain float64 definition (oracle; test infrastructure only).

What the method computes ([P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "PagedAttention分页注意力机制原理": the kernel looks each logical block up
in the block table and runs attention over the non-contiguous physical blocks;
[P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析", section 6.2: the kernel
takes out, q, k, v and block_tables) is ordinary single-query scaled
dot-product attention over each sequence's KV history.  Paging changes where
the history is stored, never the result.  So the oracle is that definition
written out:

    for sequence s with context length n, query head h, kv head g = h // G:
        z_t  = scale * sum_d q[s,h,d] * K_s[t,g,d]          t = 0 .. n-1
        o    = sum_t exp(z_t - max z) V_s[t,g,:] / sum_t exp(z_t - max z)

with G = num_heads / num_kv_heads and consecutive grouping of query heads onto
kv heads (the pages are silent on the grouping; consecutive is the reading
adopted).  Subtracting max z changes nothing mathematically; it only keeps exp
finite.  A sequence with n == 0 yields a zero row (defined so padded batches
are legal; the pages are silent).

The paged form gathers each sequence's rows into contiguous K/V first, using
only the block table: logical token t of a sequence lives in physical block
``table[t // block_size]`` at offset ``t % block_size`` ([P1]
"大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解", sections
3.2-3.3: logical block list mapped to physical blocks through the block table).
The cache layout is [num_blocks, block_size, num_kv_heads, head_dim], one pool
for K and one for V ([P2] section 2.1 gives a block's data the shape
(BLOCK_SIZE, NUM_HEADS, HEAD_SIZE)).
"""

import numpy as np

from .numerics import widen


def attend(q, K, V, scale):
    """One query row against one head's history.

    q: float64 [D]; K, V: float64 [n, D]; returns float64 [D].
    """
    q = np.asarray(q, dtype=np.float64)
    K = np.asarray(K, dtype=np.float64)
    V = np.asarray(V, dtype=np.float64)
    n = K.shape[0]
    if n == 0:
        return np.zeros(V.shape[1] if V.ndim == 2 else q.shape[0], dtype=np.float64)
    z = float(scale) * (K @ q)
    w = np.exp(z - z.max())
    return (w @ V) / w.sum()


def decode_history(q, Khist, Vhist, scale):
    """Decode one sequence from its contiguous history.

    q: float64 [Hq, D]; Khist, Vhist: float64 [n, Hkv, D].
    Query head h reads kv head h // (Hq // Hkv).  Returns float64 [Hq, D].
    """
    q = np.asarray(q, dtype=np.float64)
    Hq, D = q.shape
    Hkv = Khist.shape[1]
    if Hq % Hkv != 0:
        raise ValueError("num_heads must be a multiple of num_kv_heads")
    G = Hq // Hkv
    out = np.empty((Hq, D), dtype=np.float64)
    for h in range(Hq):
        g = h // G
        out[h] = attend(q[h], Khist[:, g, :], Vhist[:, g, :], scale)
    return out


def gather(cache, table_row, context_len, block_size):
    """Rows of one sequence, in logical order, read through its block table.

    cache: [num_blocks, block_size, Hkv, D] (storage form, any dtype);
    table_row: the sequence's physical block ids in logical order.
    Returns [context_len, Hkv, D] in the cache's storage form.
    """
    n = int(context_len)
    t = np.arange(n)
    blocks = np.asarray(table_row, dtype=np.int64)[t // block_size]
    return cache[blocks, t % block_size]


def paged_decode(q, k_cache, v_cache, block_tables, context_lens, scale,
                 block_size, dtype):
    """Decode every sequence of a batch through its block table.

    q: [S, Hq, D] storage form of ``dtype``; k_cache, v_cache:
    [num_blocks, block_size, Hkv, D] storage form; block_tables: int
    [S, max_blocks]; context_lens: int [S].  Returns float64 [S, Hq, D].
    """
    S = len(context_lens)
    out = np.empty(np.asarray(q).shape, dtype=np.float64)
    for s in range(S):
        n = int(context_lens[s])
        K = widen(gather(k_cache, block_tables[s], n, block_size), dtype)
        V = widen(gather(v_cache, block_tables[s], n, block_size), dtype)
        out[s] = decode_history(widen(q[s], dtype), K, V, scale)
    return out


def paged_decode_rows(q, k_cache, v_cache, block_tables, context_lens, scale,
                      block_size, dtype, rows):
    """Like ``paged_decode`` but only for the listed (seq, head) rows.

    Used to check sampled outputs at sizes where decoding the whole batch on
    the CPU would take too long.  Returns float64 [len(rows), D].
    """
    q = np.asarray(q)
    Hq = q.shape[1]
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    res = []
    for s, h in rows:
        n = int(context_lens[s])
        g = h // G
        K = widen(gather(k_cache[:, :, g:g + 1, :], block_tables[s], n, block_size), dtype)[:, 0, :]
        V = widen(gather(v_cache[:, :, g:g + 1, :], block_tables[s], n, block_size), dtype)[:, 0, :]
        res.append(attend(widen(q[s, h], dtype), K, V, scale))
    return np.stack(res) if res else np.zeros((0, q.shape[2]))


def paged_verify(q, k_cache, v_cache, block_tables, context_lens, scale,
                 block_size, dtype):
    """Multi-query paged attention: the target model's verification pass of
    speculative decoding ([P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与
    KV Cache 实战拆解", section 5: a draft model proposes 5-6 candidate tokens and
    the target model checks them in one parallel pass).

    q: [S, Q, Hq, D] storage form; the K/V of the Q candidate tokens are the
    last Q positions of each sequence's context (written before the call).
    Query i of sequence s sits at position p = context_lens[s] - Q + i and
    attends causally to positions 0..p of its own sequence:

        out[s, i, h] = attend(q[s, i, h], K_s[0..p, h // G], V_s[0..p, h // G])

    (Q = 1 is plain decode.)  A row with p < 0 (context shorter than Q) is a
    zero row, as an empty context is in decode.  Returns float64 [S, Q, Hq, D].
    """
    q = np.asarray(q)
    S, Q, Hq, D = q.shape
    Hkv = k_cache.shape[2]
    G = Hq // Hkv
    out = np.zeros((S, Q, Hq, D), dtype=np.float64)
    for s in range(S):
        n = int(context_lens[s])
        K = widen(gather(k_cache, block_tables[s], n, block_size), dtype)
        V = widen(gather(v_cache, block_tables[s], n, block_size), dtype)
        for i in range(Q):
            p = n - Q + i
            if p < 0:
                continue
            qi = widen(q[s, i], dtype)
            for h in range(Hq):
                out[s, i, h] = attend(qi[h], K[:p + 1, h // G], V[:p + 1, h // G], scale)
    return out
