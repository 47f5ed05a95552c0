"""Oracle block allocator with reference-counted copy-on-write, in plain Python.

TEST INFRASTRUCTURE ONLY.  It replays the same operations as the library's C++
allocator; tables, slots, reference counts and copy pairs must match exactly.

What it follows, by page and section:
  "PagedAttention and vLLM Architecture" (initnode.dev)
    section 1: a fixed pool of physical blocks allocated at startup; a per-request
      block table kept by the serving engine;
    "Why Internal Fragmentation is Bounded": a block is taken only when a new
      token overflows the current last block, so only the last block is partial;
    section 3: a prompt's blocks are shared with reference count n; a write into a
      block whose count is > 1 takes a new block from the free pool, copies the
      block, decrements the old count and repoints only that stream's table;
      later writes go to the private block.
  "PagedAttention Paper Breakdown" (fullstackaihub.com), section 2 Address
    Translation Formula (slot = T[floor(i/B)]*B + i mod B) and section 3
    (a copy-on-write trigger leaves the other streams' tables untouched).

Readings where the pages are silent: the free pool is a FIFO queue seeded by a
given order (the "random placement"), freed blocks join its tail in table order;
a forked child copies the parent's table and token count, every shared block's
count going up by one; copy-on-write happens only on a write into a shared,
partially filled last block; running out of blocks raises OutOfBlocks and
changes nothing.
"""
from collections import deque


class OutOfBlocks(RuntimeError):
    pass


class OracleAllocator:
    def __init__(self, num_blocks, block_size, free_order=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("bad allocator size")
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of 0..num_blocks-1")
        self.num_blocks = num_blocks
        self.B = block_size
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.tables = {}
        self.ntokens = {}
        self.cow_count = 0

    # [fullstackaihub] section 2: PhysicalAddr = T[floor(i/B)]*B + (i mod B)
    def slot(self, seq_id, i):
        table = self.tables[seq_id]
        return table[i // self.B] * self.B + i % self.B

    def _take(self):
        blk = self.free.popleft()
        assert self.ref[blk] == 0
        self.ref[blk] = 1
        return blk

    def add_seq(self, seq_id, num_tokens):
        """New sequence holding num_tokens tokens; returns their slots."""
        if seq_id in self.tables:
            raise ValueError("sequence exists")
        if num_tokens < 0:
            raise ValueError("negative token count")
        need = -(-num_tokens // self.B)
        if need > len(self.free):
            raise OutOfBlocks()
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.ntokens[seq_id] = num_tokens
        return [self.slot(seq_id, i) for i in range(num_tokens)]

    def fork(self, parent, child):
        """Child shares every block of the parent (each count + 1)."""
        if parent not in self.tables or child in self.tables:
            raise ValueError("bad fork")
        self.tables[child] = list(self.tables[parent])
        self.ntokens[child] = self.ntokens[parent]
        for blk in self.tables[child]:
            self.ref[blk] += 1

    def append_slot(self, seq_id):
        """Slot for one new token; returns (slot, (src, dst) or None)."""
        if seq_id not in self.tables:
            raise ValueError("unknown sequence")
        table = self.tables[seq_id]
        i = self.ntokens[seq_id]
        cow = None
        if i % self.B == 0:
            # the last block is full (or there is none): take a fresh block
            if not self.free:
                raise OutOfBlocks()
            table.append(self._take())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                # write into a shared block: copy-on-write
                if not self.free:
                    raise OutOfBlocks()
                dst = self._take()
                self.ref[last] -= 1
                table[-1] = dst
                cow = (last, dst)
                self.cow_count += 1
        self.ntokens[seq_id] = i + 1
        return self.slot(seq_id, i), cow

    def free_seq(self, seq_id):
        if seq_id not in self.tables:
            raise ValueError("unknown sequence")
        for blk in self.tables.pop(seq_id):
            self.ref[blk] -= 1
            if self.ref[blk] == 0:
                self.free.append(blk)
        del self.ntokens[seq_id]

    def block_table(self, seq_id):
        return list(self.tables[seq_id])

    def num_free(self):
        return len(self.free)

    def waste_tokens(self, seq_id):
        """Unused slots in the sequence's table (only its last block can be partial)."""
        return len(self.tables[seq_id]) * self.B - self.ntokens[seq_id]
