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
