"""Reserved versus used KV slots over a request trace (oracle; test
infrastructure only).

[P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section on
the memory bottleneck: contiguous per-request pre-allocation leaves reserved
memory idle that no other request can use; paging holds only the blocks a
sequence has filled, wasting at most the tail of its last block.

Definitions used here (token slots; bytes are a constant multiple):
* paged, one step: reserved = bs x |distinct physical blocks in any live
  table|; used = |distinct slots table[p // bs] * bs + p % bs over live
  sequences and positions p < context length|.
* contiguous, one step: every running sequence reserves its context at
  admission + max_new_tokens; used = its context length.
* static batching: arrival-order batches of B members; each member reserves
  the batch's longest prompt + longest output for the batch's duration
  (its longest output, in steps); at decode step k a member uses
  prompt + min(k, its output).
Waste = 1 - (sum over steps of used) / (sum over steps of reserved).
"""


def paged_step(bm):
    """(reserved slots, used slots) of the live sequences of a block manager."""
    bs = bm.block_size
    blocks, slots = set(), set()
    for seq, table in bm.tables.items():
        blocks.update(table)
        for p in range(bm.ctx[seq]):
            slots.add(table[p // bs] * bs + p % bs)
    return len(blocks) * bs, len(slots)


def contiguous_trace(steps, max_new_tokens):
    """steps: list of (running ids, context lengths) per step."""
    first, reserved, used = {}, 0, 0
    for run, ctx in steps:
        for s, n in zip(run, ctx):
            first.setdefault(s, n - 1)     # the context before this step's token
            reserved += first[s] + max_new_tokens
            used += n
    return reserved, used


def static_trace(members, batch, max_steps):
    """members: (prompt tokens, output tokens) in arrival order."""
    reserved = used = t = 0
    for i in range(0, len(members), batch):
        grp = members[i:i + batch]
        longest_prompt = max(p for p, _ in grp)
        longest_out = max(o for _, o in grp)
        for k in range(1, longest_out + 1):
            if t == max_steps:
                return reserved, used
            for p, o in grp:
                reserved += longest_prompt + longest_out
                used += p + min(k, o)
            t += 1
    return reserved, used
