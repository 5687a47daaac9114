"""Oracle: host block allocator with reference counts (Python model).

TEST INFRASTRUCTURE ONLY — see ``oracle/__init__.py``.

What the pages fix
------------------
* Blocks are fixed-size and handed out on demand: a sequence gets a new block
  only when its last one is full ("PagedAttention" concept card, section
  带来的能力: one new block every 16 tokens; "什么是 LLM 中的分页注意力", section
  使用分页注意力: block 2 is allocated when block 1 is full, block 3 when block 2
  is full).  A sequence of ``n`` tokens therefore holds ``ceil(n / bs)`` blocks
  and wastes ``ceil(n / bs) * bs - n`` slots, all in its last block (worked
  example: 3 blocks of 4 for 10 tokens, 2 slots wasted).
* Blocks can be shared; each carries a reference count, a fork increments the
  count of every block it shares, and a block whose count reaches 0 is
  reclaimed ("深入解析 PagedAttention", sections 核心创新 and 多序列共享;
  concept card, section 实现要点).
* Before a sequence writes into a block it still shares, that block is copied
  (copy on write) so the sibling's prefix is not modified (concept card,
  section 实现要点).

Readings where the pages are silent (listed in the design notes):

* Copy on write happens at append time iff the sequence's last block is
  partially filled and its refcount is ``> 1``: a fresh block is taken, the
  pair ``(src, dst)`` is reported for the device copy, ``refcount(src)`` drops
  by one, and the sequence's table points at ``dst``.  With ``n`` forks, the
  first ``n - 1`` writers copy; the last one then holds refcount 1 and writes
  in place.  A full shared last block needs no copy: the next token starts a
  fresh block.
* The free list is a LIFO stack.  Initially pops return ``0, 1, 2, ...``; with
  a non-zero ``shuffle_seed`` they return a Fisher–Yates permutation of
  ``range(num_blocks)`` driven by splitmix64 (Steele, Lea & Flood, "Fast
  splittable pseudorandom number generators", OOPSLA 2014), index drawn as
  ``next() % (i + 1)`` for ``i = n-1 .. 1``.  An explicit initial pop order may
  be given instead.  Freed blocks are pushed in table order.
* ``internal_waste_slots`` sums ``len(table) * bs - num_tokens`` over live
  sequences (per sequence, as in the worked example).
* Every failing call (out of blocks, unknown or duplicate id) leaves the
  state unchanged.
"""

from __future__ import annotations

_MASK64 = (1 << 64) - 1


class OutOfBlocks(Exception):
    """No free physical block is left; the allocator state is unchanged."""


def splitmix64_stream(seed):
    """Yield the splitmix64 sequence for ``seed`` (64-bit unsigned outputs)."""
    state = seed & _MASK64
    while True:
        state = (state + 0x9E3779B97F4A7C15) & _MASK64
        z = state
        z = ((z ^ (z >> 30)) * 0xBF58476D1CE4E5B9) & _MASK64
        z = ((z ^ (z >> 27)) * 0x94D049BB133111EB) & _MASK64
        yield z ^ (z >> 31)


def _initial_pop_order(num_blocks, shuffle_seed):
    order = list(range(num_blocks))
    if shuffle_seed:
        gen = splitmix64_stream(shuffle_seed)
        for i in range(num_blocks - 1, 0, -1):
            j = next(gen) % (i + 1)
            order[i], order[j] = order[j], order[i]
    return order


class RefAllocator:
    """Reference-counted physical block allocator for a paged KV pool."""

    def __init__(self, num_blocks, block_size, shuffle_seed=0, pop_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if pop_order is None:
            pop_order = _initial_pop_order(num_blocks, shuffle_seed)
        pop_order = [int(x) for x in pop_order]
        if sorted(pop_order) != list(range(num_blocks)):
            raise ValueError("pop_order must be a permutation of range(num_blocks)")
        # LIFO stack: the last element is popped first.
        self.free = list(reversed(pop_order))
        self.ref = [0] * num_blocks
        self.tables = {}   # seq_id -> list of physical block ids
        self.ntok = {}     # seq_id -> number of tokens

    # -- queries -------------------------------------------------------------
    def num_free(self):
        return len(self.free)

    def refcount(self, block):
        return self.ref[block]

    def block_table(self, seq_id):
        return list(self.tables[seq_id]), self.ntok[seq_id]

    def seq_slots(self, seq_id):
        """Slot of every token: token t sits in block table[t // bs] at offset t % bs."""
        table, n = self.tables[seq_id], self.ntok[seq_id]
        return [table[t // self.block_size] * self.block_size + t % self.block_size for t in range(n)]

    def internal_waste_slots(self):
        return sum(len(t) * self.block_size - self.ntok[s] for s, t in self.tables.items())

    # -- mutations -----------------------------------------------------------
    def _pop(self):
        b = self.free.pop()
        self.ref[b] = 1
        return b

    def add_seq(self, seq_id, num_tokens):
        """Register a sequence holding ``num_tokens`` tokens: ``ceil(n/bs)`` fresh blocks."""
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id} already exists")
        if num_tokens < 0:
            raise ValueError("num_tokens must be >= 0")
        need = -(-num_tokens // self.block_size)
        if need > len(self.free):
            raise OutOfBlocks(f"need {need} blocks, {len(self.free)} free")
        self.tables[seq_id] = [self._pop() for _ in range(need)]
        self.ntok[seq_id] = num_tokens

    def fork(self, parent_id, child_id):
        """The child shares every block of the parent; each block's refcount +1."""
        if parent_id not in self.tables:
            raise KeyError(f"unknown sequence {parent_id}")
        if child_id in self.tables:
            raise KeyError(f"sequence {child_id} already exists")
        table = list(self.tables[parent_id])
        for b in table:
            self.ref[b] += 1
        self.tables[child_id] = table
        self.ntok[child_id] = self.ntok[parent_id]

    def append_slot(self, seq_id):
        """Reserve the slot of the sequence's next token.

        Returns ``(slot, cow_src, cow_dst)``; ``cow_src == cow_dst == -1`` when
        no copy is needed.  ``slot = phys * bs + offset``.
        """
        if seq_id not in self.tables:
            raise KeyError(f"unknown sequence {seq_id}")
        table = self.tables[seq_id]
        pos = self.ntok[seq_id]
        off = pos % self.block_size
        src = dst = -1
        if off == 0:
            # no block yet, or the last block is full: take a fresh one
            if not self.free:
                raise OutOfBlocks("no free block for a new block")
            phys = self._pop()
            table.append(phys)
        else:
            last = table[-1]
            if self.ref[last] > 1:
                if not self.free:
                    raise OutOfBlocks("no free block for copy-on-write")
                phys = self._pop()
                self.ref[last] -= 1
                table[-1] = phys
                src, dst = last, phys
            else:
                phys = last
        self.ntok[seq_id] = pos + 1
        return phys * self.block_size + off, src, dst

    def truncate(self, seq_id, num_tokens):
        """Keep the first ``num_tokens`` tokens; blocks past ceil(n/bs) are released in
        table order (speculative rollback, concept card section 已知局限)."""
        if seq_id not in self.tables:
            raise KeyError(f"unknown sequence {seq_id}")
        if not 0 <= num_tokens <= self.ntok[seq_id]:
            raise ValueError("num_tokens out of range")
        keep = -(-num_tokens // self.block_size)
        table = self.tables[seq_id]
        for b in table[keep:]:
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del table[keep:]
        self.ntok[seq_id] = num_tokens

    def beam_select(self, seq_ids, parent_idx):
        """Beam i continues from beam parent_idx[i] (beam search shares the blocks before
        the branch point: concept card section 带来的能力).  New references first, then
        the old tables are released, beam 0 first, each in table order."""
        seq_ids = [int(x) for x in seq_ids]
        if len(set(seq_ids)) != len(seq_ids) or any(s not in self.tables for s in seq_ids):
            raise KeyError("beam ids must be distinct live sequences")
        if any(not 0 <= int(p) < len(seq_ids) for p in parent_idx):
            raise ValueError("parent index out of range")
        new = [(list(self.tables[seq_ids[int(p)]]), self.ntok[seq_ids[int(p)]]) for p in parent_idx]
        for table, _ in new:
            for b in table:
                self.ref[b] += 1
        for sid in seq_ids:
            for b in self.tables[sid]:
                self.ref[b] -= 1
                if self.ref[b] == 0:
                    self.free.append(b)
        for sid, (table, n) in zip(seq_ids, new):
            self.tables[sid] = table
            self.ntok[sid] = n

    def free_seq(self, seq_id):
        """Drop the sequence; blocks whose refcount reaches 0 return to the free list."""
        if seq_id not in self.tables:
            raise KeyError(f"unknown sequence {seq_id}")
        for b in self.tables.pop(seq_id):
            self.ref[b] -= 1
            if self.ref[b] == 0:
                self.free.append(b)
        del self.ntok[seq_id]
