"""Iteration-level (continuous) batching, plain Python model (oracle; test
infrastructure only).

Policy ([P1] "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解",
section 2.2, Scheduler.schedule; [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "连续批处理Continuous Batching配置"), one call of ``step()``:

1. Finished sequences leave the batch and return their blocks.
2. Admission, first-come first-served: with a block budget equal to the free
   block count, take the head of the waiting queue while its required blocks
   fit the budget, charge the budget, and stop at the first request that does
   not fit (it stays at the head; the pages' pseudocode stops with ``break``).
   ``required = ceil(unshared_tokens / block_size) + 1`` (room for the first
   generated token; +1 more when the request forks a parallel-sampling child).
   The number of running sequences is also capped (``max_running``, the
   pages' max-num-seqs).  An admitted request's prompt is placed: a
   prefix-sharing request forks the resident prefix holder (shares its blocks
   by reference) and appends its own tokens; any other request allocates its
   tokens.  A request with a fork child then forks it (the child shares every
   block, including a partly filled last one).
3. Every running sequence, in admission order, reserves the slot of its next
   token.  When the pool is exhausted, the most recently admitted running
   sequence is preempted: its blocks are freed and it goes back to the FRONT of
   the waiting queue, keeping its progress; on re-admission its whole history
   is written again (recompute).  ([P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析",
   section 3.2 names preemptive scheduling without an algorithm; this is the
   reading adopted.)  Copy-on-write pairs from the block manager are reported.
4. Each running sequence has generated one more token; it finishes once it has
   generated ``output_len`` tokens (removed at the start of the next step).

``step()`` returns a record of everything the device must do and everything a
checker compares: cache writes (seq, position, slot) in issue order, CoW
pairs, admitted / preempted / finished ids, and the running batch with its
context lengths.  ``ops`` holds the writes and CoW copies interleaved in
issue order: a copy must see every earlier write to its source block and none
of the later ones, so the device has to apply them in that order.  When a
preemption frees blocks, every op of the step that targets a freed block (a
write into it, a copy into it) is dropped from the record: that work is dead,
and a freed block can be taken again later in the same step, so keeping it
would list one slot twice.  Within a step every slot is written at most once.

Preemption by swap (``preempt="swap"``, with a ``SwappingBlockManager``; [P3]
"大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
"生产部署注意事项": KV cache moved out to CPU memory when GPU memory runs short
and back in later), readings adopted:

* A victim whose privately held blocks fit the host pool is swapped out
  instead of freed: ("so", gpu, cpu) copies join ``ops`` right there, the
  victim keeps its progress and joins the FIFO swapped queue.  Its writes of
  this step stay (the copies carry them out).  When the host pool is short,
  the victim is recomputed as above.
* Before admission, swapped sequences come back first, in queue order, each
  needing its host blocks + 1 (its next token) from the step's budget:
  ("si", cpu, gpu) copies, and it rejoins the running batch.  New requests are
  admitted only once the swapped queue is empty.
* A recompute preemption drops the dead ops of the step as above ("so" ops
  target host blocks and always stay).  A preemption happens only when no
  GPU block is free, so at that moment every block a swap-out freed earlier
  in the step has been taken again: only the recomputed victim's own ops
  become dead.  Ops run in issue order; consecutive writes form one launch,
  and within one such run every slot is distinct.

Admission through the prefix cache (``prefix_cache=True``, with a
prefix-caching manager; [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置",
section "Prefix Caching前缀复用优化": a request whose prompt begins with cached
KV references those blocks and skips their prefill), readings adopted:

* Requests carry their prompt token ids; a prefix-sharing request's tokens
  are the system prefix's ids (given to the scheduler) followed by its own.
  The token a sequence generates at position p comes from ``token_fn(seq,
  p)``, an input (it stands in for the sampled token; the tests pass the
  counter-based generator of the input module, which the C++ scheduler
  implements from the same published definition).
* The prefix holder's full blocks must be the cached blocks of the prefix
  ids (checked at construction).  Then a prefix-sharing admission finds all
  of them, and no admission takes more blocks than the budget charges it.
* Admission calls ``allocate_prefix`` with the sequence's whole token history
  (prompt, and on re-admission the tokens generated so far) and records cache
  writes only past the cached part.  The budget charge is unchanged (it does
  not count on hits).  Decode appends go through ``append_token``.
* A recompute preemption frees the victim as usual; then every block that an
  op of this step targets and that is now unreferenced but still named is
  forgotten (name dropped, back to the free list) before the dead ops are
  dropped: a block whose writes are abandoned must not be found by a later
  lookup.  A named block written in earlier steps keeps its name and waits
  on the evictable list, so a re-admission finds it again.
"""

from dataclasses import dataclass, field

from .block_manager import NoBlocks, ceil_div


@dataclass
class Request:
    seq_id: int
    prompt_len: int            # tokens of the request's own (unshared) prompt
    output_len: int            # tokens to generate before finishing
    shares_prefix: bool = False
    fork_child: int = -1       # id of a parallel-sampling child, -1 for none
    fork_output_len: int = 0
    tokens: list = None        # own prompt token ids (prefix-cache admission)


@dataclass
class _Seq:
    seq_id: int
    output_len: int
    shares_prefix: bool
    history: int               # tokens held (prefix included) while running
    generated: int = 0
    fork_child: int = -1
    fork_output_len: int = 0
    forked: bool = False
    is_child: bool = False
    tokens: list = None        # whole token history (prefix-cache admission)


@dataclass
class StepRecord:
    finished: list = field(default_factory=list)
    admitted: list = field(default_factory=list)
    preempted: list = field(default_factory=list)
    writes: list = field(default_factory=list)      # (seq, position, slot)
    cow: list = field(default_factory=list)         # (src, dst)
    ops: list = field(default_factory=list)         # ("w", seq, pos, slot) | ("c", src, dst)
                                                    # | ("so", gpu, cpu) | ("si", cpu, gpu)
    swapped_out: list = field(default_factory=list)
    swapped_in: list = field(default_factory=list)
    running: list = field(default_factory=list)     # seq ids, admission order
    context_lens: list = field(default_factory=list)

    def write(self, seq, pos, slot):
        self.writes.append((seq, pos, slot))
        self.ops.append(("w", seq, pos, slot))

    def copy(self, src, dst):
        self.cow.append((src, dst))
        self.ops.append(("c", src, dst))

    def swap(self, kind, a, b):
        self.ops.append((kind, a, b))

    def drop_dead(self, bm):
        """Remove ops whose target GPU block is back on the free list."""
        bs = bm.block_size

        def live(op):
            if op[0] == "so":                     # targets a host block
                return True
            return bm.ref[op[3] // bs if op[0] == "w" else op[2]] > 0

        self.ops = [op for op in self.ops if live(op)]
        self.writes = [(o[1], o[2], o[3]) for o in self.ops if o[0] == "w"]
        self.cow = [(o[1], o[2]) for o in self.ops if o[0] == "c"]


class Scheduler:
    def __init__(self, bm, max_running, prefix_seq=-1, preempt="recompute", prefix_cache=False,
                 prefix_tokens=None, token_fn=None):
        if preempt not in ("recompute", "swap"):
            raise ValueError(preempt)
        self.prefix_cache = bool(prefix_cache)
        self.prefix_tokens = [int(t) for t in (prefix_tokens or [])]
        self.token_fn = token_fn
        if self.prefix_cache and token_fn is None:
            raise ValueError("prefix-cache admission needs the generated tokens")
        if self.prefix_cache and prefix_seq >= 0:
            # every full block of the holder must be the cached block of these
            # ids, so a sharer finds them all and stays within its charge
            bs, table = bm.block_size, bm.tables.get(prefix_seq)
            ok = table is not None and bm.ctx[prefix_seq] == len(self.prefix_tokens)
            ok = ok and not (hasattr(bm, "swapped") and bm.swapped(prefix_seq))
            for j in range(len(self.prefix_tokens) // bs if ok else 0):
                ok = ok and bm.cache.get(tuple(self.prefix_tokens[:(j + 1) * bs])) == table[j]
            if not ok:
                raise ValueError("the prefix holder's blocks are not cached under these token ids")
        self.bm = bm
        self.preempt = preempt
        self.swapped = []          # swapped-out sequences, FIFO
        self.max_running = int(max_running)
        self.prefix_seq = prefix_seq
        self.prefix_len = bm.context_len(prefix_seq) if prefix_seq >= 0 else 0
        self.waiting = []          # list of _Seq, FCFS order
        self.running = []          # list of _Seq, admission order

    def add_request(self, req):
        if req.shares_prefix and self.prefix_seq < 0:
            raise ValueError("prefix-sharing request without a prefix holder")
        base = self.prefix_len if req.shares_prefix else 0
        s = _Seq(req.seq_id, req.output_len, req.shares_prefix, base + req.prompt_len, 0, req.fork_child,
                 req.fork_output_len)
        if self.prefix_cache:
            own = [int(t) for t in req.tokens]
            if len(own) != req.prompt_len:
                raise ValueError("prompt tokens and prompt length disagree")
            s.tokens = (list(self.prefix_tokens) if req.shares_prefix else []) + own
        self.waiting.append(s)

    def _unshared(self, s):
        return s.history - (self.prefix_len if s.shares_prefix else 0)

    def _required(self, s):
        need = ceil_div(self._unshared(s), self.bm.block_size) + 1
        if s.fork_child >= 0 and not s.forked:
            need += 1
        return need

    def _admit(self, s, rec):
        bm = self.bm
        if self.prefix_cache:
            cached = bm.allocate_prefix(s.seq_id, s.tokens[:s.history])
            for pos, slot in enumerate(bm.slots(s.seq_id, cached, s.history - cached), start=cached):
                rec.write(s.seq_id, pos, slot)
        elif s.shares_prefix:
            bm.fork(self.prefix_seq, s.seq_id)
            for pos in range(self.prefix_len, s.history):
                slot, src, dst = bm.append_slot(s.seq_id)
                if src >= 0:
                    rec.copy(src, dst)
                rec.write(s.seq_id, pos, slot)
        else:
            bm.allocate(s.seq_id, s.history)
            for pos, slot in enumerate(bm.slots(s.seq_id, 0, s.history)):
                rec.write(s.seq_id, pos, slot)
        self.running.append(s)
        rec.admitted.append(s.seq_id)
        if s.fork_child >= 0 and not s.forked:
            s.forked = True
            bm.fork(s.seq_id, s.fork_child)
            child = _Seq(s.fork_child, s.fork_output_len, s.shares_prefix,
                         s.history, 0, is_child=True)
            if self.prefix_cache:
                child.tokens = list(s.tokens[:s.history])
            self.running.append(child)
            rec.admitted.append(child.seq_id)

    def _preempt_last(self, rec):
        victim = self.running.pop()
        bm = self.bm
        if self.preempt == "swap":
            try:
                pairs = bm.swap_out(victim.seq_id)
            except NoBlocks:
                pairs = None
            if pairs is not None:
                for g, c in pairs:
                    rec.swap("so", g, c)
                self.swapped.append(victim)
                rec.swapped_out.append(victim.seq_id)
                rec.preempted.append(victim.seq_id)
                return victim
        bm.free(victim.seq_id)
        if self.prefix_cache:
            # blocks this step targets that are now unreferenced but still named:
            # their writes are about to be dropped, so their names must go too
            bs = bm.block_size
            seen = set()
            for op in rec.ops:
                if op[0] == "so":
                    continue
                b = op[3] // bs if op[0] == "w" else op[2]
                if b in seen:
                    continue
                seen.add(b)
                if bm.ref[b] == 0 and b in bm.name:
                    bm.forget(b)
        rec.drop_dead(bm)
        self.waiting.insert(0, victim)
        rec.preempted.append(victim.seq_id)
        return victim

    def step(self):
        rec = StepRecord()
        bm = self.bm
        # 1. finish
        keep = []
        for s in self.running:
            if s.generated >= s.output_len:
                bm.free(s.seq_id)
                rec.finished.append(s.seq_id)
            else:
                keep.append(s)
        self.running = keep
        # 2. swapped sequences come back first, then admission (FCFS, stop at the
        # first request that does not fit), only once none is left swapped out
        budget = bm.num_free
        while self.swapped and len(self.running) < self.max_running:
            s = self.swapped[0]
            need = sum(bm.on_cpu[s.seq_id]) + 1
            if need > budget:
                break
            self.swapped.pop(0)
            budget -= need
            for c, g in bm.swap_in(s.seq_id):
                rec.swap("si", c, g)
            self.running.append(s)
            rec.swapped_in.append(s.seq_id)
        while not self.swapped and self.waiting and budget > 0 and len(self.running) < self.max_running:
            s = self.waiting[0]
            need = self._required(s)
            if need > budget:
                break
            extra = 1 if (s.fork_child >= 0 and not s.forked) else 0
            if len(self.running) + 1 + extra > self.max_running:
                break
            self.waiting.pop(0)
            budget -= need
            self._admit(s, rec)
        # 3. reserve the next token's slot for every running sequence
        i = 0
        while i < len(self.running):
            s = self.running[i]
            try:
                if self.prefix_cache:
                    tok = int(self.token_fn(s.seq_id, s.history))
                    slot, src, dst = bm.append_token(s.seq_id, tok)
                else:
                    slot, src, dst = bm.append_slot(s.seq_id)
            except NoBlocks:
                victim = self._preempt_last(rec)
                if victim is s:
                    continue          # the sequence itself was preempted
                continue              # retry the same sequence
            if src >= 0:
                rec.copy(src, dst)
            rec.write(s.seq_id, s.history, slot)
            if self.prefix_cache:
                del s.tokens[s.history:]
                s.tokens.append(tok)
            s.history += 1
            s.generated += 1
            i += 1
        rec.running = [s.seq_id for s in self.running]
        rec.context_lens = [s.history for s in self.running]
        return rec
