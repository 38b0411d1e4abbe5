"""Oracle model of the paged KV-cache block manager -- TEST INFRASTRUCTURE ONLY.

Plain Python, one step at a time, in the order the pages describe.  Only tests/,
the smoke check and bench.py's CPU-baseline leg may use it.  It shares no code
with the GPU library's C++ block manager; the two are compared bit for bit.

Sources ("What problem does PagedAttention solve, and what is continuous
batching?" = page 1; "PagedAttention & Continuous Batching" = page 2;
"Continuous Batching & Paged Attention" = page 3):

* page 1, "How PagedAttention works": the KV cache lives in fixed-size blocks
  (16 tokens in the example); a request of 50 tokens needs four logical blocks,
  three full and one holding two tokens; a block table maps logical block number
  to physical block; the allocator can take any free block; the last partially
  filled block wastes at most one block.
* page 1, same section: blocks may be shared (beam candidates with a common
  prefix); when one diverges, copy-on-write gives it a private block for the
  changed portion.
* page 1, "A concrete memory example": when a request finishes, its blocks go
  back to the pool at once and a new request can use them.
* page 3, "Paged attention borrows a trick from operating systems": when a
  request grows, the server attaches another block.

Readings where the pages leave a step open (each listed in the design notes):

1. "any free block": a LIFO stack over a given order of the block ids; the
   first id of ``order`` is handed out first.
2. alloc on an empty stack fails with OutOfBlocks and changes nothing.
3. free(b) decrements b's reference count; at zero b is pushed back (so the
   next alloc reuses it); freeing a block whose count is zero is DoubleFree.
4. appending one token to a sequence of length L: if L % B == 0 a new block is
   attached; else if the tail block is shared (count > 1) it is copied on write:
   a new block is taken, the pair (tail, new) recorded, the tail's count
   decremented and the table entry replaced.  The slot written is
   table[L // B] * B + L % B; L becomes L + 1.
5. a batch of appends runs in batch order, token by token; if the pool runs out
   part way, the whole call fails and nothing changes.
6. retiring a sequence decrements its blocks in logical order; forking one
   increments its blocks in logical order.

Prefix caching (page 1, same section: "Prefix caching can use a similar idea";
page 2, "If you remember three things": shared prefixes are shared blocks).  The
pages give no lookup, so the reading taken is:

7. a full block can be registered under a caller-supplied 64-bit key (a hash
   chain of its tokens and all tokens before it); a key maps to one block and a
   block has at most one key; registering an existing key or a registered block
   changes nothing.
8. a registered block whose count drops to zero is not pushed on the free
   stack: it joins the back of an evictable queue (least recently released at
   the front) and keeps its key.
9. alloc takes the top of the free stack; only when the stack is empty does it
   evict the front of the queue (the key is forgotten) and hand that block out.
10. a new sequence built from keys walks them in order and shares each
   registered block (count + 1, leaving the queue if it was there) until the
   first miss; its length is then (hits x B).

Preemption with swap (page 1, "The senior-level nuance" and "What happens when
the KV cache is full?": a full pool must queue, preempt, offload or reject):

11. swapping a sequence out copies its blocks, in logical order, to host memory
   and then drops one reference on each of them (logical order, as a retire
   does); the sequence keeps its id and length but owns no block.
12. swapping it back in takes ceil(L / B) blocks from the allocator one after
   the other (as appends would) and copies the data back in logical order; if
   the pool cannot supply them all, nothing changes.
"""
from __future__ import annotations

import copy
from collections import OrderedDict


class OutOfBlocks(Exception):
    pass


class DoubleFree(Exception):
    pass


class InvalidArgument(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks: int, block_size: int, order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidArgument("num_blocks and block_size must be positive")
        order = list(range(num_blocks)) if order is None else [int(b) for b in order]
        if sorted(order) != list(range(num_blocks)):
            raise InvalidArgument("order must be a permutation of the block ids")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free_stack = list(reversed(order))   # top of stack = end of list = order[0]
        self.refcount = [0] * num_blocks
        self.tables: dict[int, list[int]] = {}
        self.lengths: dict[int, int] = {}
        self.next_seq = 0
        self.key_of: dict[int, int] = {}            # block -> key (registered blocks)
        self.block_of: dict[int, int] = {}          # key -> block
        self.evictable: OrderedDict = OrderedDict()  # registered blocks with count 0, oldest first
        self.swapped: set[int] = set()              # sequences whose blocks are in host memory

    # ---- blocks --------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free_stack) + len(self.evictable)

    def alloc(self) -> int:
        if self.free_stack:
            b = self.free_stack.pop()
        elif self.evictable:
            b, _ = self.evictable.popitem(last=False)
            del self.block_of[self.key_of.pop(b)]
        else:
            raise OutOfBlocks()
        self.refcount[b] = 1
        return b

    def free(self, b: int) -> None:
        self._check_block(b)
        if self.refcount[b] == 0:
            raise DoubleFree(b)
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            if b in self.key_of:
                self.evictable[b] = None
            else:
                self.free_stack.append(b)

    def incref(self, b: int) -> None:
        self._check_block(b)
        if self.refcount[b] == 0:
            raise InvalidArgument(f"block {b} is free")
        self.refcount[b] += 1

    def _check_block(self, b: int) -> None:
        if not 0 <= b < self.num_blocks:
            raise InvalidArgument(f"block {b} out of range")

    # ---- sequences -----------------------------------------------------------
    def seq_add(self) -> int:
        sid = self.next_seq
        self.next_seq += 1
        self.tables[sid] = []
        self.lengths[sid] = 0
        return sid

    def seq_fork(self, parent: int) -> int:
        if parent not in self.tables or parent in self.swapped:
            raise InvalidArgument(parent)
        child = self.seq_add()
        for b in self.tables[parent]:
            self.incref(b)
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        return child

    def seq_free(self, sid: int) -> None:
        if sid not in self.tables:
            raise InvalidArgument(sid)
        for b in self.tables[sid]:
            self.free(b)
        del self.tables[sid]
        del self.lengths[sid]
        self.swapped.discard(sid)

    def _append_one(self, sid: int, cow_pairs: list) -> int:
        B = self.block_size
        L = self.lengths[sid]
        table = self.tables[sid]
        if L % B == 0:
            table.append(self.alloc())
        else:
            tail = table[-1]
            if self.refcount[tail] > 1:
                new = self.alloc()
                cow_pairs.append((tail, new))
                self.refcount[tail] -= 1
                table[-1] = new
        slot = table[L // B] * B + L % B
        self.lengths[sid] = L + 1
        return slot

    def reserve_slots(self, seq_ids, ntok):
        """Append ntok[i] tokens to seq_ids[i], in batch order.

        Returns (slot_mapping, cow_pairs); on OutOfBlocks nothing changes.
        """
        seq_ids = [int(s) for s in seq_ids]
        ntok = [int(n) for n in ntok]
        if len(seq_ids) != len(ntok) or len(set(seq_ids)) != len(seq_ids):
            raise InvalidArgument("seq_ids must be distinct and match ntok")
        for s, n in zip(seq_ids, ntok):
            if s not in self.tables or n < 0 or s in self.swapped:
                raise InvalidArgument(s)
        saved = copy.deepcopy((self.free_stack, self.refcount, self.tables, self.lengths, self.key_of,
                               self.block_of, self.evictable))
        slots, cow = [], []
        try:
            for s, n in zip(seq_ids, ntok):
                for _ in range(n):
                    slots.append(self._append_one(s, cow))
        except OutOfBlocks:
            (self.free_stack, self.refcount, self.tables, self.lengths, self.key_of, self.block_of,
             self.evictable) = saved
            raise
        return slots, cow

    # ---- prefix caching --------------------------------------------------------
    def register(self, sid: int, keys) -> int:
        """Register the first len(keys) blocks of sid (all full) under keys; returns
        how many were newly registered."""
        if sid not in self.tables:
            raise InvalidArgument(sid)
        keys = [int(k) for k in keys]
        if len(keys) * self.block_size > self.lengths[sid]:
            raise InvalidArgument("only full blocks can be registered")
        new = 0
        for b, k in zip(self.tables[sid], keys):
            if k in self.block_of or b in self.key_of:
                continue
            self.block_of[k] = b
            self.key_of[b] = k
            new += 1
        return new

    def seq_add_cached(self, keys):
        """New sequence sharing the registered blocks of its leading keys; (sid, hits)."""
        sid = self.seq_add()
        table = self.tables[sid]
        for k in keys:
            b = self.block_of.get(int(k))
            if b is None:
                break
            if self.refcount[b] == 0:
                del self.evictable[b]
            self.refcount[b] += 1
            table.append(b)
        self.lengths[sid] = len(table) * self.block_size
        return sid, len(table)

    # ---- preemption with swap ---------------------------------------------------
    def swap_out(self, sid: int):
        """Returns the blocks whose contents go to host memory (logical order)."""
        if sid not in self.tables or sid in self.swapped:
            raise InvalidArgument(sid)
        blocks = list(self.tables[sid])
        for b in blocks:
            self.free(b)
        self.tables[sid] = []
        self.swapped.add(sid)
        return blocks

    def swap_in(self, sid: int):
        """Returns the new blocks the host copy is written back to (logical order)."""
        if sid not in self.swapped:
            raise InvalidArgument(sid)
        n = -(-self.lengths[sid] // self.block_size)
        saved = copy.deepcopy((self.free_stack, self.refcount, self.key_of, self.block_of, self.evictable))
        try:
            blocks = [self.alloc() for _ in range(n)]
        except OutOfBlocks:
            self.free_stack, self.refcount, self.key_of, self.block_of, self.evictable = saved
            raise
        self.tables[sid] = blocks
        self.swapped.discard(sid)
        return blocks

    # ---- views ---------------------------------------------------------------
    def table(self, sid: int) -> list[int]:
        return list(self.tables[sid])

    def length(self, sid: int) -> int:
        return self.lengths[sid]

    def dense_tables(self, seq_ids, max_blocks: int, pad: int = -1):
        """Dense [n][max_blocks] table (padded with ``pad``) and lengths for seq_ids."""
        rows, lens = [], []
        for s in seq_ids:
            t = self.tables[int(s)]
            if len(t) > max_blocks:
                raise InvalidArgument("max_blocks too small")
            rows.append(t + [pad] * (max_blocks - len(t)))
            lens.append(self.lengths[int(s)])
        return rows, lens
