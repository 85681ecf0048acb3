"""Pure-Python model of the paged block allocator -- test infrastructure only.

What the pages fix:

* "Paged attention in LLMs", section "The fix: stop demanding one
  continuous run": a request takes a fixed-size block when it needs one and
  another, from wherever space is free, when that block fills.
* same page, "Keeping track: the block table": each request owns a table
  mapping its logical block index to a physical block.
* same page, "Sharing blocks", and the quiz page's table rows "Prefix
  sharing across requests: share physical pages" and "Beam search / best of
  N: copy on write blocks": several tables may point at one physical block;
  a write into a shared block first copies it.
* the quiz page's analogy: blocks are returned as a request finishes.

What the pages leave open, and the reading taken here:

* Free-list policy: a LIFO stack.  A fresh allocator pops blocks in the
  order ``initial_order`` (default 0, 1, 2, ...).  A freed block is pushed on
  top; a finished request's blocks are pushed in table order.
* Copy-on-write trigger: appending into a partially filled last block whose
  reference count is above 1 takes a new block, records the pair
  (src, dst), drops one reference from src and points this request's table
  at dst.  Full shared blocks are never written, so they are never copied.
  Of k requests sharing a partial block, the first k-1 writers copy and the
  last one writes in place.
* A request's append is all-or-nothing: when the free list runs dry the
  whole call fails and nothing changes.
"""

import copy


class OutOfBlocks(Exception):
    """Raised when an append needs more free blocks than the pool holds."""


class BlockAllocator:
    def __init__(self, num_blocks, block_size, initial_order=None):
        if initial_order is None:
            initial_order = range(num_blocks)
        order = [int(b) for b in initial_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("initial_order must be a permutation of the blocks")
        self.num_blocks = num_blocks
        self.block_size = block_size
        # top of the stack is the end of the list
        self._free = list(reversed(order))
        self._refcount = [0] * num_blocks
        self._tables = {}
        self._lens = {}

    # -- queries ---------------------------------------------------------
    def num_free(self):
        return len(self._free)

    def seq_len(self, seq_id):
        return self._lens[seq_id]

    def block_table(self, seq_id):
        return list(self._tables[seq_id])

    def refcount(self, block):
        return self._refcount[block]

    def free_list(self):
        """Free blocks in the order the next pops return them."""
        return list(reversed(self._free))

    def refcounts(self):
        return list(self._refcount)

    def seq_ids(self):
        return sorted(self._tables)

    # -- mutations -------------------------------------------------------
    def add_seq(self, seq_id):
        if seq_id in self._tables:
            raise KeyError(f"sequence {seq_id} exists")
        self._tables[seq_id] = []
        self._lens[seq_id] = 0

    def fork(self, parent, child):
        """Child shares every block of the parent ("Sharing blocks")."""
        if child in self._tables:
            raise KeyError(f"sequence {child} exists")
        self._tables[child] = list(self._tables[parent])
        self._lens[child] = self._lens[parent]
        for block in self._tables[child]:
            self._refcount[block] += 1

    def _pop(self):
        if not self._free:
            raise OutOfBlocks()
        return self._free.pop()

    def _append_one(self, seq_id, slots, cow_pairs):
        table = self._tables[seq_id]
        pos = self._lens[seq_id]
        offset = pos % self.block_size
        if offset == 0:
            block = self._pop()
            self._refcount[block] = 1
            table.append(block)
        else:
            block = table[-1]
            if self._refcount[block] > 1:
                fresh = self._pop()
                cow_pairs.append((block, fresh))
                self._refcount[block] -= 1
                self._refcount[fresh] = 1
                table[-1] = fresh
                block = fresh
        slots.append(block * self.block_size + offset)
        self._lens[seq_id] = pos + 1

    def append(self, seq_id, num_tokens):
        """Append tokens to one request; returns (slots, cow_pairs)."""
        return self.append_batch([seq_id], num_tokens)

    def append_batch(self, seq_ids, num_tokens):
        """Append ``num_tokens`` to each request, requests in the given order.

        Returns (slots, cow_pairs): slots in (request, token) order, and the
        copy-on-write pairs in the order they arose.  On OutOfBlocks the
        allocator is left exactly as it was before the call.
        """
        saved = copy.deepcopy((self._free, self._refcount, self._tables, self._lens))
        slots, cow_pairs = [], []
        try:
            for seq_id in seq_ids:
                for _ in range(num_tokens):
                    self._append_one(seq_id, slots, cow_pairs)
        except OutOfBlocks:
            self._free, self._refcount, self._tables, self._lens = saved
            raise
        return slots, cow_pairs

    def free_seq(self, seq_id):
        """Drop a request; blocks whose count reaches 0 return to the free list."""
        table = self._tables.pop(seq_id)
        del self._lens[seq_id]
        for block in table:
            self._refcount[block] -= 1
            if self._refcount[block] == 0:
                self._free.append(block)
