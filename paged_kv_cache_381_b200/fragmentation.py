"""KV memory reserved versus used: paged blocks against contiguous reservation.

Contiguous per-request KV reservation against paging:
"大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
"大模型推理显存瓶颈分析" (each request pre-allocates one contiguous region
sized for its maximum length; the unused part cannot serve other requests);
"大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解",
section 1 (padding under static batching often wastes over 40%) and the
table of section 8 (KV-cache fragmentation of 42% for static batching, 35%
for continuous batching, under 5% with PagedAttention).

Three layouts are accounted over the same request trace, step by step, as
token slots (multiply by 2 * num_kv_heads * head_dim * element size for
bytes; the ratio does not depend on it):

* paged -- the native scheduler and block manager run the trace; each step
  `pa_bm_usage` gives the blocks held and their filled slots (a block shared
  by several sequences is counted once);
* contiguous -- the same admitted timeline, but every running sequence holds
  a private contiguous region of (its prompt, system prefix included) +
  `max_new_tokens` slots from admission to finish;
* static -- requests in arrival order form fixed batches of `batch` requests;
  a batch reserves, for each member, the batch's longest prompt + longest
  output, and holds it until its longest member finishes.

waste = 1 - sum over steps of used slots / sum over steps of reserved slots.
"""

from . import workloads as wl


def paged_usage(tc=wl.TRACE, seed=0, steps=None, pool_blocks=None):
    """Run the native scheduler over the trace; per step (held blocks, filled
    slots, running sequence ids, their context lengths).  `pool_blocks`
    defaults to a pool large enough that nothing is preempted."""
    import paged_kv_cache_381_b200 as pa
    reqs = wl.make_trace_requests(tc, seed)
    steps = tc.steps if steps is None else steps
    if pool_blocks is None:
        peak = sum(-(-(tc.prefix_len + q.prompt_len + q.output_len) // tc.block_size) + 1 for q in reqs)
        peak += sum(-(-(tc.prefix_len + q.prompt_len + q.fork_output_len) // tc.block_size) + 1
                    for q in reqs if q.fork_child >= 0)
        pool_blocks = peak + -(-tc.prefix_len // tc.block_size)
    bm = pa.BlockManager(pool_blocks, tc.block_size)
    bm.allocate(wl.PREFIX_SEQ, tc.prefix_len)
    sch = pa.Scheduler(bm, tc.max_running, wl.PREFIX_SEQ)
    for q in reqs:
        sch.add_request(q.seq_id, q.prompt_len, q.output_len, q.shares_prefix, q.fork_child, q.fork_output_len)
    out = []
    for _ in range(steps):
        rec = sch.step()
        held, filled = bm.usage()
        out.append((held, filled, rec["running"], rec["context_lens"]))
    return out


def _members(tc, reqs):
    """(prompt with prefix, output) per sequence id, children included."""
    out = {}
    for q in reqs:
        pre = tc.prefix_len if q.shares_prefix else 0
        out[q.seq_id] = (pre + q.prompt_len, q.output_len)
        if q.fork_child >= 0:
            out[q.fork_child] = (pre + q.prompt_len, q.fork_output_len)
    return out


def study(tc=wl.TRACE, seed=0, steps=None, max_new_tokens=(2048, 1024, 512), batch=None):
    """Waste of the three layouts over the trace (see the module docstring).
    Contiguous reservation is reported for each max_new_tokens, and as
    "exact" for a reservation of each sequence's true output length (the best
    a contiguous layout could do)."""
    bs = tc.block_size
    rows = paged_usage(tc, seed, steps)
    reqs = wl.make_trace_requests(tc, seed)
    mem = _members(tc, reqs)
    held_slots = sum(h * bs for h, _, _, _ in rows)
    filled = sum(f for _, f, _, _ in rows)
    res = {"steps": len(rows), "block_size": bs,
           "paged": {"reserved": held_slots, "used": filled, "waste": 1.0 - filled / held_slots}}
    # contiguous: the context before a sequence's first step is its context at admission
    first = {}
    for _, _, run, ctx in rows:
        for s, n in zip(run, ctx):
            first.setdefault(s, n - 1)
    used = sum(sum(ctx) for _, _, _, ctx in rows)
    cont = {}
    for label in list(max_new_tokens) + ["exact"]:
        reserved = 0
        for _, _, run, _ in rows:
            for s in run:
                reserved += first[s] + (mem[s][1] if label == "exact" else label)
        cont[str(label)] = {"reserved": reserved, "used": used, "waste": 1.0 - used / reserved}
    res["contiguous"] = cont
    # static batching over the same sequences in arrival order, children right after their parent
    order = []
    for q in reqs:
        order.append(mem[q.seq_id])
        if q.fork_child >= 0:
            order.append(mem[q.fork_child])
    B = tc.max_running if batch is None else batch
    s_res = s_used = t = 0
    for i in range(0, len(order), B):
        grp = order[i:i + B]
        pad = max(p for p, _ in grp) + max(o for _, o in grp)
        for k in range(1, max(o for _, o in grp) + 1):
            if t == len(rows):
                break
            s_res += pad * len(grp)
            s_used += sum(p + min(k, o) for p, o in grp)
            t += 1
        if t == len(rows):
            break
    res["static"] = {"reserved": s_res, "used": s_used, "waste": 1.0 - s_used / s_res, "batch": B}
    return res


if __name__ == "__main__":
    import json
    print(json.dumps(study(), indent=1))
