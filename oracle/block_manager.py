"""Block-manager bookkeeping, plain Python model (oracle; test infrastructure only).

Policy, from the pages, with the readings adopted where they are silent:

* Pool of equal-size physical blocks, kept on a free list ([P1]
  "大模型推理引擎高频优化：连续批处理、PagedAttention 与 KV Cache 实战拆解", section 3.3:
  blocks are taken with ``free_blocks.pop()``, i.e. from the END of the list;
  [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
  "PagedAttention分页注意力机制原理": requests take blocks from the free pool on
  demand and give them back when they finish).  The initial list order is a
  parameter (a seeded permutation stands for "shuffled physical ids").
* ``allocate(seq, n)`` takes ceil(n / block_size) blocks, popped in logical
  order ([P1] section 3.3, allocate with ceil_div).
* A per-block reference count ([P2] "vLLM推理加速框架：PagedAttention与连续批处理技术解析",
  section 2.1: each Block carries ref_count).
* ``fork(parent, child)`` shares every block of the parent by reference
  (prefix sharing, [P3] same section: sequences referencing the same physical
  block share prefix KV; parallel sampling, [P2] section 1.1).
* ``append_slot(seq)`` reserves the slot of the next token: a new block is taken
  only when the last one is full ([P1] section 3.3, append_token); if the last
  block is shared (ref > 1) it is first copied to a fresh block
  (copy-on-write, [P2] section 2.2) and the (src, dst) pair is reported so the
  caller can copy the block's contents.
* ``free(seq)`` walks the table in logical order, decrements each block's
  count and pushes blocks that reach zero onto the free list (push order is
  the reading adopted; the pages only say blocks are returned).

Operations that cannot be satisfied raise ``NoBlocks`` and leave the state
unchanged; misuse raises ``InvalidArg``.
"""


class NoBlocks(Exception):
    """Free list cannot satisfy the request (state unchanged)."""


class InvalidArg(Exception):
    """Unknown / duplicate sequence id or malformed argument."""


def ceil_div(a, b):
    return -(-int(a) // int(b))


class BlockManager:
    def __init__(self, num_blocks, block_size, initial_free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidArg("num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if initial_free_order is None else [int(b) for b in initial_free_order]
        if sorted(order) != list(range(num_blocks)):
            raise InvalidArg("initial free order must be a permutation of the pool")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        self.free_list = order          # pop() takes the last element
        self.ref = [0] * self.num_blocks
        self.tables = {}                # seq id -> list of physical ids, logical order
        self.ctx = {}                   # seq id -> tokens held

    # -- queries ---------------------------------------------------------------
    @property
    def num_free(self):
        return len(self.free_list)

    @property
    def num_used(self):
        return self.num_blocks - len(self.free_list)

    def block_table(self, seq):
        if seq not in self.tables:
            raise InvalidArg(f"unknown sequence {seq}")
        return list(self.tables[seq])

    def context_len(self, seq):
        if seq not in self.ctx:
            raise InvalidArg(f"unknown sequence {seq}")
        return self.ctx[seq]

    def slots(self, seq, start, count):
        """Slots of logical positions [start, start + count) of ``seq``."""
        table = self.tables[seq]
        bs = self.block_size
        if start < 0 or start + count > len(table) * bs:
            raise InvalidArg("positions outside the sequence's blocks")
        return [table[p // bs] * bs + p % bs for p in range(start, start + count)]

    # -- operations ------------------------------------------------------------
    def allocate(self, seq, num_tokens):
        if seq in self.tables:
            raise InvalidArg(f"sequence {seq} already exists")
        if num_tokens < 0:
            raise InvalidArg("negative token count")
        need = ceil_div(num_tokens, self.block_size)
        if need > len(self.free_list):
            raise NoBlocks(f"need {need} blocks, {len(self.free_list)} free")
        blocks = [self.free_list.pop() for _ in range(need)]
        for b in blocks:
            self.ref[b] = 1
        self.tables[seq] = blocks
        self.ctx[seq] = int(num_tokens)
        return list(blocks)

    def fork(self, parent, child):
        if parent not in self.tables:
            raise InvalidArg(f"unknown sequence {parent}")
        if child in self.tables:
            raise InvalidArg(f"sequence {child} already exists")
        blocks = list(self.tables[parent])
        for b in blocks:
            self.ref[b] += 1
        self.tables[child] = blocks
        self.ctx[child] = self.ctx[parent]

    def append_slot(self, seq):
        """Reserve the next token's slot.  Returns (slot, cow_src, cow_dst)."""
        if seq not in self.tables:
            raise InvalidArg(f"unknown sequence {seq}")
        table = self.tables[seq]
        bs = self.block_size
        pos = self.ctx[seq]
        cow_src = cow_dst = -1
        if pos % bs == 0:
            # last block full (or none yet): take a fresh block, never a copy
            if not self.free_list:
                raise NoBlocks("no free block for a new token")
            b = self.free_list.pop()
            self.ref[b] = 1
            table.append(b)
        else:
            last = table[-1]
            if self.ref[last] > 1:
                if not self.free_list:
                    raise NoBlocks("no free block for copy-on-write")
                b = self.free_list.pop()
                self.ref[b] = 1
                self.ref[last] -= 1
                table[-1] = b
                cow_src, cow_dst = last, b
        self.ctx[seq] = pos + 1
        slot = table[pos // bs] * bs + pos % bs
        return slot, cow_src, cow_dst

    def free(self, seq):
        if seq not in self.tables:
            raise InvalidArg(f"unknown sequence {seq}")
        for b in self.tables[seq]:
            if self.ref[b] <= 0:
                raise AssertionError("reference count underflow")
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free_list.append(b)
        del self.tables[seq]
        del self.ctx[seq]

    # -- invariants ------------------------------------------------------------
    def check(self):
        """Raise AssertionError unless every bookkeeping invariant holds."""
        held = {}
        for seq, table in self.tables.items():
            assert len(table) == ceil_div(self.ctx[seq], self.block_size), seq
            for b in table:
                held[b] = held.get(b, 0) + 1
        for b in range(self.num_blocks):
            assert self.ref[b] == held.get(b, 0), (b, self.ref[b], held.get(b, 0))
        free = set(self.free_list)
        assert len(free) == len(self.free_list), "duplicate on free list"
        assert free.isdisjoint(held.keys()), "block both free and held"
        assert free | set(held.keys()) == set(range(self.num_blocks)), "block lost"
        assert sum(self.ref) == sum(len(t) for t in self.tables.values())


class PrefixCachingBlockManager(BlockManager):
    """Block manager with a prefix cache (oracle; test infrastructure only).

    [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
    "Prefix Caching前缀复用优化": when a new request begins with a prefix whose KV
    is already cached, it references those blocks instead of computing them
    again.  Readings adopted where the page is silent:

    * Only FULL blocks are cached, each under the whole token prefix that ends
      with it: block j of a table is named by ``tuple(tokens[:(j + 1) * bs])``.
      Two requests hit the same block exactly when their first (j + 1) * bs
      tokens agree, so a hit never reuses KV computed for other tokens.
    * A block is named only if every earlier block of its table is the block
      the cache names for that earlier prefix (the cache is a tree grown from
      the first block), and only if its prefix and the block are not named yet.
    * ``allocate_prefix`` walks the prompt's full blocks from the first and
      stops at the first prefix the cache does not hold; it references the
      blocks found and takes fresh ones for the rest.  Partly filled blocks are
      never shared through the cache.
    * A named block whose count reaches zero is not put on the free list; it
      waits on an evictable list, oldest first, still counted as free.  A
      fresh block comes from the free list while it has one, else the oldest
      evictable block is taken and its name dropped (least recently used).
    * ``free`` walks the table as the plain manager does; the named blocks that
      reach zero join the evictable list last block first, so a deeper block
      is always evicted before the block it extends.
    * ``allocate`` and ``append_slot`` give no token ids: such a sequence
      names no further blocks.  ``append_token`` gives the id and names the
      block it fills.
    """

    def __init__(self, num_blocks, block_size, initial_free_order=None):
        super().__init__(num_blocks, block_size, initial_free_order)
        self.cache = {}          # token prefix (tuple) -> block
        self.name = {}           # block -> token prefix
        self.evictable = []      # named blocks with count zero, oldest first
        self.tokens = {}         # seq id -> token ids held, or None when unknown
        self.hits = 0
        self.lookups = 0

    @property
    def num_free(self):
        return len(self.free_list) + len(self.evictable)

    @property
    def num_used(self):
        return self.num_blocks - self.num_free

    @property
    def num_cached(self):
        return len(self.name)

    def _take(self):
        if self.free_list:
            return self.free_list.pop()
        b = self.evictable.pop(0)
        del self.cache[self.name.pop(b)]
        return b

    def _key(self, toks, j):
        """Name of block j of a table holding ``toks``: the whole prefix ending with it."""
        return tuple(toks[:(j + 1) * self.block_size])

    def _name(self, seq, j):
        """Name block j of seq's table, if the rules above allow it."""
        table, toks = self.tables[seq], self.tokens[seq]
        bs = self.block_size
        if toks is None or len(toks) < (j + 1) * bs:
            return
        for i in range(j):
            if self.cache.get(self._key(toks, i)) != table[i]:
                return
        key = self._key(toks, j)
        if key in self.cache or table[j] in self.name:
            return
        self.cache[key] = table[j]
        self.name[table[j]] = key

    def allocate(self, seq, num_tokens):
        if seq in self.tables:
            raise InvalidArg(f"sequence {seq} already exists")
        if num_tokens < 0:
            raise InvalidArg("negative token count")
        need = ceil_div(num_tokens, self.block_size)
        if need > self.num_free:
            raise NoBlocks(f"need {need} blocks, {self.num_free} free")
        blocks = [self._take() for _ in range(need)]
        for b in blocks:
            self.ref[b] = 1
        self.tables[seq] = blocks
        self.ctx[seq] = int(num_tokens)
        self.tokens[seq] = [] if num_tokens == 0 else None
        return list(blocks)

    def allocate_prefix(self, seq, tokens):
        """New sequence holding ``tokens``; returns how many leading tokens are cached."""
        if seq in self.tables:
            raise InvalidArg(f"sequence {seq} already exists")
        toks = [int(t) for t in tokens]
        bs = self.block_size
        nfull = len(toks) // bs
        found, probed = [], 0
        for j in range(nfull):
            probed += 1
            b = self.cache.get(self._key(toks, j))
            if b is None:
                break
            found.append(b)
        need = ceil_div(len(toks), bs) - len(found)
        if need > self.num_free - sum(1 for b in found if b in self.evictable):
            raise NoBlocks(f"need {need} blocks")
        self.lookups += probed
        self.hits += len(found)
        for b in found:
            if b in self.evictable:
                self.evictable.remove(b)
            self.ref[b] += 1
        table = list(found)
        self.tables[seq] = table
        self.ctx[seq] = len(toks)
        self.tokens[seq] = toks
        for j in range(len(found), ceil_div(len(toks), bs)):
            b = self._take()
            self.ref[b] = 1
            table.append(b)
            self._name(seq, j)
        return len(found) * bs

    def fork(self, parent, child):
        super().fork(parent, child)
        t = self.tokens[parent]
        self.tokens[child] = None if t is None else list(t)

    def forget(self, b):
        """Drop the name of an unreferenced cached block and free it (its K/V is
        not to be trusted, e.g. writes into it were abandoned)."""
        if self.ref[b] != 0 or b not in self.name:
            raise InvalidArg(f"block {b} is not an unreferenced cached block")
        self.evictable.remove(b)
        del self.cache[self.name.pop(b)]
        self.free_list.append(b)

    def _append(self, seq, token):
        if seq not in self.tables:
            raise InvalidArg(f"unknown sequence {seq}")
        table = self.tables[seq]
        bs = self.block_size
        pos = self.ctx[seq]
        cow_src = cow_dst = -1
        if pos % bs == 0 or self.ref[table[-1]] > 1:
            if self.num_free == 0:
                raise NoBlocks("no block for the next token")
            b = self._take()
            self.ref[b] = 1
            if pos % bs == 0:
                table.append(b)
            else:                                   # copy-on-write of a shared last block
                cow_src, cow_dst = table[-1], b
                self.ref[table[-1]] -= 1
                table[-1] = b
        self.ctx[seq] = pos + 1
        toks = self.tokens[seq]
        if toks is not None and token is not None:
            toks.append(int(token))
        else:
            self.tokens[seq] = None
        if (pos + 1) % bs == 0:
            self._name(seq, pos // bs)
        return table[pos // bs] * bs + pos % bs, cow_src, cow_dst

    def append_slot(self, seq):
        return self._append(seq, None)

    def append_token(self, seq, token):
        return self._append(seq, token)

    def free(self, seq):
        if seq not in self.tables:
            raise InvalidArg(f"unknown sequence {seq}")
        named = []
        for b in self.tables[seq]:
            if self.ref[b] <= 0:
                raise AssertionError("reference count underflow")
            self.ref[b] -= 1
            if self.ref[b] == 0:
                if b in self.name:
                    named.append(b)
                else:
                    self.free_list.append(b)
        self.evictable.extend(reversed(named))
        del self.tables[seq], self.ctx[seq], self.tokens[seq]

    def check(self):
        held = {}
        for seq, table in self.tables.items():
            assert len(table) == ceil_div(self.ctx[seq], self.block_size), seq
            for b in table:
                held[b] = held.get(b, 0) + 1
        for b in range(self.num_blocks):
            assert self.ref[b] == held.get(b, 0), (b, self.ref[b], held.get(b, 0))
        free, ev = set(self.free_list), set(self.evictable)
        assert len(free) == len(self.free_list) and len(ev) == len(self.evictable), "duplicate"
        assert not (free & ev) and not (free & held.keys()) and not (ev & held.keys()), "block in two places"
        assert free | ev | set(held) == set(range(self.num_blocks)), "block lost"
        assert ev <= set(self.name), "evictable block without a name"
        assert not (free & set(self.name)), "named block on the free list"
        assert {self.cache[k]: k for k in self.cache} == self.name, "cache and names disagree"
        for key, b in self.cache.items():
            assert len(key) % self.block_size == 0 and len(key) > 0


class SwappingBlockManager(BlockManager):
    """Block manager with a host (CPU) swap pool (oracle; test infrastructure only).

    [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM连续批处理配置", section
    "生产部署注意事项": when GPU memory runs short, the KV cache of some requests
    is moved out to CPU memory and moved back once GPU memory is free again.
    Readings adopted where the page is silent:

    * The host pool holds ``num_cpu_blocks`` blocks of the same shape, on its
      own free list (taken from the end, like the GPU list).
    * ``swap_out(seq)`` moves every block the sequence holds ALONE (count 1)
      to a host block, in logical order, and returns the GPU block it leaves
      to the free list (logical order); blocks it shares (count > 1) stay on
      the GPU and the sequence keeps its reference, since their contents
      remain resident for the other holders.  Returns the (gpu, cpu) copies
      to run BEFORE the freed GPU blocks are reused.  All or nothing: with too
      few host blocks, NoBlocks and no change.
    * ``swap_in(seq)`` takes a fresh GPU block for each host block of the
      sequence, in logical order, returns the host blocks to their list, and
      returns the (cpu, gpu) copies.  All or nothing on GPU blocks.
    * A swapped-out sequence cannot append or fork; ``free`` releases its host
      blocks (logical order) and its shared GPU references.
    """

    def __init__(self, num_blocks, block_size, num_cpu_blocks, initial_free_order=None):
        super().__init__(num_blocks, block_size, initial_free_order)
        self.num_cpu_blocks = int(num_cpu_blocks)
        self.cpu_free = list(range(self.num_cpu_blocks))
        self.on_cpu = {}                 # seq id -> list of bools per logical block (swapped sequences)

    def swapped(self, seq):
        return seq in self.on_cpu

    def swap_out(self, seq):
        if seq not in self.tables or seq in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is not resident")
        table = self.tables[seq]
        alone = [j for j, b in enumerate(table) if self.ref[b] == 1]
        if len(alone) > len(self.cpu_free):
            raise NoBlocks(f"need {len(alone)} host blocks, {len(self.cpu_free)} free")
        loc = [False] * len(table)
        pairs = []
        for j in alone:
            g = table[j]
            c = self.cpu_free.pop()
            pairs.append((g, c))
            self.ref[g] = 0
            self.free_list.append(g)
            table[j] = c
            loc[j] = True
        self.on_cpu[seq] = loc
        return pairs

    def swap_in(self, seq):
        if seq not in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is not swapped out")
        table, loc = self.tables[seq], self.on_cpu[seq]
        need = sum(loc)
        if need > len(self.free_list):
            raise NoBlocks(f"need {need} blocks, {len(self.free_list)} free")
        pairs = []
        for j, here in enumerate(loc):
            if here:
                c = table[j]
                g = self.free_list.pop()
                self.ref[g] = 1
                pairs.append((c, g))
                self.cpu_free.append(c)
                table[j] = g
        del self.on_cpu[seq]
        return pairs

    def fork(self, parent, child):
        if parent in self.on_cpu:
            raise InvalidArg(f"sequence {parent} is swapped out")
        super().fork(parent, child)

    def append_slot(self, seq):
        if seq in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is swapped out")
        return super().append_slot(seq)

    def free(self, seq):
        if seq not in self.on_cpu:
            return super().free(seq)
        for b, here in zip(self.tables[seq], self.on_cpu[seq]):
            if here:
                self.cpu_free.append(b)
            else:
                if self.ref[b] <= 0:
                    raise AssertionError("reference count underflow")
                self.ref[b] -= 1
                if self.ref[b] == 0:
                    self.free_list.append(b)
        del self.tables[seq], self.ctx[seq], self.on_cpu[seq]

    def check(self):
        held, cpu_held = {}, []
        for seq, table in self.tables.items():
            assert len(table) == ceil_div(self.ctx[seq], self.block_size), seq
            loc = self.on_cpu.get(seq, [False] * len(table))
            for b, here in zip(table, loc):
                if here:
                    cpu_held.append(b)
                else:
                    held[b] = held.get(b, 0) + 1
        for b in range(self.num_blocks):
            assert self.ref[b] == held.get(b, 0), (b, self.ref[b], held.get(b, 0))
        free = set(self.free_list)
        assert len(free) == len(self.free_list) and free.isdisjoint(held)
        assert free | set(held) == set(range(self.num_blocks)), "block lost"
        assert len(set(cpu_held)) == len(cpu_held), "host block held twice"
        cf = set(self.cpu_free)
        assert len(cf) == len(self.cpu_free) and cf.isdisjoint(cpu_held)
        assert cf | set(cpu_held) == set(range(self.num_cpu_blocks)), "host block lost"


class PrefixSwappingBlockManager(PrefixCachingBlockManager):
    """Prefix cache and host swap pool together (oracle; test infrastructure only).

    The two sections of [P3] "大模型推理显存优化实战：PagedAttention机制原理与vLLM
    连续批处理配置" ("Prefix Caching前缀复用优化", "生产部署注意事项") at once.
    Everything of PrefixCachingBlockManager holds; swap follows
    SwappingBlockManager with these readings where the two meet:

    * ``swap_out`` copies every block the sequence holds alone to a host
      block, in logical order.  Such a block that the cache names keeps its
      name and joins the evictable list (last block first, as ``free`` does),
      so its K/V stays reusable on the GPU until it is evicted; the others go
      to the free list.  The sequence remembers each named block and its name.
    * ``swap_in`` needs as many free GPU blocks (free list + evictable) as the
      sequence has host blocks, all or nothing.  In logical order, a
      remembered block that the cache still names by the same name is taken
      back (off the evictable list if it is there; another holder may have
      referenced it meanwhile) with no copy; any other host block gets a
      fresh block (which may evict) and a (cpu, gpu) copy.  Host blocks go
      back to their list.  Blocks filled in this way are not named again.
    * ``free`` of a swapped-out sequence returns its host blocks and drops its
      GPU references; named blocks reaching zero join the evictable list last
      block first.
    """

    def __init__(self, num_blocks, block_size, num_cpu_blocks, initial_free_order=None):
        super().__init__(num_blocks, block_size, initial_free_order)
        self.num_cpu_blocks = int(num_cpu_blocks)
        self.cpu_free = list(range(self.num_cpu_blocks))
        self.on_cpu = {}         # seq id -> per logical block, True = host block
        self.left = {}           # seq id -> per logical block, (GPU block, name) left in the cache, or None

    def swapped(self, seq):
        return seq in self.on_cpu

    def swap_out(self, seq):
        if seq not in self.tables or seq in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is not resident")
        table = self.tables[seq]
        alone = [j for j, b in enumerate(table) if self.ref[b] == 1]
        if len(alone) > len(self.cpu_free):
            raise NoBlocks(f"need {len(alone)} host blocks, {len(self.cpu_free)} free")
        loc, left, named, pairs = [False] * len(table), [None] * len(table), [], []
        for j in alone:
            g = table[j]
            c = self.cpu_free.pop()
            pairs.append((g, c))
            self.ref[g] = 0
            if g in self.name:
                named.append(g)
                left[j] = (g, self.name[g])
            else:
                self.free_list.append(g)
            table[j] = c
            loc[j] = True
        self.evictable.extend(reversed(named))
        self.on_cpu[seq], self.left[seq] = loc, left
        return pairs

    def swap_in(self, seq):
        if seq not in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is not swapped out")
        table, loc, left = self.tables[seq], self.on_cpu[seq], self.left[seq]
        need = sum(loc)
        if need > self.num_free:
            raise NoBlocks(f"need {need} blocks, {self.num_free} free")
        pairs = []
        for j, here in enumerate(loc):
            if not here:
                continue
            c = table[j]
            kept = left[j]
            if kept is not None and self.cache.get(kept[1]) == kept[0]:
                g = kept[0]                     # still cached under the same name: no copy
                if g in self.evictable:
                    self.evictable.remove(g)
                self.ref[g] += 1
            else:
                g = self._take()
                self.ref[g] = 1
                pairs.append((c, g))
            self.cpu_free.append(c)
            table[j] = g
        del self.on_cpu[seq], self.left[seq]
        return pairs

    def fork(self, parent, child):
        if parent in self.on_cpu:
            raise InvalidArg(f"sequence {parent} is swapped out")
        super().fork(parent, child)

    def _append(self, seq, token):
        if seq in self.on_cpu:
            raise InvalidArg(f"sequence {seq} is swapped out")
        return super()._append(seq, token)

    def free(self, seq):
        if seq not in self.on_cpu:
            return super().free(seq)
        named = []
        for b, here in zip(self.tables[seq], self.on_cpu[seq]):
            if here:
                self.cpu_free.append(b)
                continue
            if self.ref[b] <= 0:
                raise AssertionError("reference count underflow")
            self.ref[b] -= 1
            if self.ref[b] == 0:
                if b in self.name:
                    named.append(b)
                else:
                    self.free_list.append(b)
        self.evictable.extend(reversed(named))
        del self.tables[seq], self.ctx[seq], self.tokens[seq], self.on_cpu[seq], self.left[seq]

    def check(self):
        held, cpu_held = {}, []
        for seq, table in self.tables.items():
            assert len(table) == ceil_div(self.ctx[seq], self.block_size), seq
            loc = self.on_cpu.get(seq, [False] * len(table))
            for b, here in zip(table, loc):
                if here:
                    cpu_held.append(b)
                else:
                    held[b] = held.get(b, 0) + 1
        for b in range(self.num_blocks):
            assert self.ref[b] == held.get(b, 0), (b, self.ref[b], held.get(b, 0))
        free, ev = set(self.free_list), set(self.evictable)
        assert len(free) == len(self.free_list) and len(ev) == len(self.evictable), "duplicate"
        assert not (free & ev) and not (free & held.keys()) and not (ev & held.keys()), "block in two places"
        assert free | ev | set(held) == set(range(self.num_blocks)), "block lost"
        assert ev <= set(self.name), "evictable block without a name"
        assert not (free & set(self.name)), "named block on the free list"
        assert {self.cache[k]: k for k in self.cache} == self.name, "cache and names disagree"
        assert len(set(cpu_held)) == len(cpu_held), "host block held twice"
        cf = set(self.cpu_free)
        assert len(cf) == len(self.cpu_free) and cf.isdisjoint(cpu_held)
        assert cf | set(cpu_held) == set(range(self.num_cpu_blocks)), "host block lost"
