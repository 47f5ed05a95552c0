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
    (a copy-on-write trigger leaves the other streams' tables untouched);
    "Paper Methods": shared prefix caching kept in a radix tree.

Readings where the pages are silent: the free pool is a FIFO queue seeded by a
given order (the "random placement"), freed blocks join its tail in table order;
a forked child copies the parent's table and token count, every shared block's
count going up by one; copy-on-write happens only on a write into a shared,
partially filled last block; running out of blocks raises OutOfBlocks and
changes nothing (a batch of appends included).

Host tier ([fullstackaihub] "Engineering Limitations": CPU-GPU block swapping
under memory pressure; the pages give no policy, only the mechanism).  Read as: a
separate pool of host blocks with its own FIFO free queue; swapping a sequence out
gives each of its blocks, in table order, a host block and drops the sequence's
reference to the device block; swapping in takes device blocks as any allocation
does and frees the host blocks; a swapped-out sequence is only held, never used.

Prefix cache (the pages name the radix tree only).  The tree is read at block
granularity: each node is one full physical block, labelled by the B token ids it
holds and hanging under the node of the block before it, so the path from the root
spells the token prefix.  Adding a prompt by its token ids reuses the blocks along
the longest matching path (count + 1), takes fresh blocks for its other full blocks
and hangs them under that path, and gives a partial last block a fresh private
block.  A cached block whose count reaches zero stays in the tree, unreferenced.
Blocks come from the free queue first; when it is empty, the unreferenced cached
block released earliest among those with no child in the tree is removed from the
tree and reused.
"""
import copy
from collections import OrderedDict, deque


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
        self.tree = {}            # (parent block or -1, token ids of the block) -> block
        self.key_of = {}          # cached block -> its key in the tree
        self.nchildren = {}       # cached block -> number of cached children
        self.unreferenced = OrderedDict()   # cached blocks with count 0, earliest release first
        self.host_free = deque()  # host tier: free host blocks
        self.num_host_blocks = 0
        self.on_host = set()      # sequences swapped out (their tables hold host blocks)

    # [fullstackaihub] section 2: PhysicalAddr = T[floor(i/B)]*B + (i mod B)
    def slot(self, seq_id, i):
        table = self.tables[seq_id]
        return table[i // self.B] * self.B + i % self.B

    def available(self):
        return len(self.free) + len(self.unreferenced)

    def _take(self):
        if self.free:
            blk = self.free.popleft()
        else:
            blk = next(b for b in self.unreferenced if self.nchildren[b] == 0)
            key = self.key_of.pop(blk)
            del self.tree[key]
            del self.nchildren[blk]
            del self.unreferenced[blk]
            if key[0] >= 0:
                self.nchildren[key[0]] -= 1
        assert self.ref[blk] == 0
        self.ref[blk] = 1
        return blk

    def _hold(self, blk):
        if self.ref[blk] == 0:
            del self.unreferenced[blk]
        self.ref[blk] += 1

    def _release(self, blk):
        self.ref[blk] -= 1
        if self.ref[blk] == 0:
            if blk in self.key_of:
                self.unreferenced[blk] = None
            else:
                self.free.append(blk)

    def add_seq(self, seq_id, num_tokens):
        """New sequence holding num_tokens tokens; returns their slots."""
        if seq_id in self.tables:
            raise ValueError("sequence exists")
        if num_tokens < 0:
            raise ValueError("negative token count")
        need = -(-num_tokens // self.B)
        if need > self.available():
            raise OutOfBlocks()
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.ntokens[seq_id] = num_tokens
        return [self.slot(seq_id, i) for i in range(num_tokens)]

    def add_seq_cached(self, seq_id, token_ids):
        """New sequence with these token ids, reusing the cached blocks of its longest
        cached full-block prefix.  Returns (slots, number of tokens already cached)."""
        if seq_id in self.tables:
            raise ValueError("sequence exists")
        tokens = [int(t) for t in token_ids]
        n, B = len(tokens), self.B
        full = [tuple(tokens[j * B:(j + 1) * B]) for j in range(n // B)]
        hits, parent = [], -1
        for blk_tokens in full:
            blk = self.tree.get((parent, blk_tokens))
            if blk is None:
                break
            hits.append(blk)
            parent = blk
        need = len(full) - len(hits) + (1 if n % B else 0)
        if need > self.available() - sum(1 for b in hits if self.ref[b] == 0):
            raise OutOfBlocks()
        table = []
        for blk in hits:
            self._hold(blk)
            table.append(blk)
        for blk_tokens in full[len(hits):]:
            blk = self._take()
            key = (parent, blk_tokens)
            self.tree[key] = blk
            self.key_of[blk] = key
            self.nchildren[blk] = 0
            if parent >= 0:
                self.nchildren[parent] += 1
            table.append(blk)
            parent = blk
        if n % B:
            table.append(self._take())
        self.tables[seq_id] = table
        self.ntokens[seq_id] = n
        return [self.slot(seq_id, i) for i in range(n)], len(hits) * B

    def fork(self, parent, child):
        """Child shares every block of the parent (each count + 1)."""
        if parent not in self.tables or parent in self.on_host or child in self.tables:
            raise ValueError("bad fork")
        self.tables[child] = list(self.tables[parent])
        self.ntokens[child] = self.ntokens[parent]
        for blk in self.tables[child]:
            self._hold(blk)

    def append_slot(self, seq_id):
        """Slot for one new token; returns (slot, (src, dst) or None)."""
        if seq_id not in self.tables or seq_id in self.on_host:
            raise ValueError("unknown or swapped-out sequence")
        table = self.tables[seq_id]
        i = self.ntokens[seq_id]
        cow = None
        if i % self.B == 0:
            # the last block is full (or there is none): take a fresh block
            if not self.available():
                raise OutOfBlocks()
            table.append(self._take())
        else:
            last = table[-1]
            if self.ref[last] > 1:
                # write into a shared block: copy-on-write
                if not self.available():
                    raise OutOfBlocks()
                dst = self._take()
                self._release(last)
                table[-1] = dst
                cow = (last, dst)
                self.cow_count += 1
        self.ntokens[seq_id] = i + 1
        return self.slot(seq_id, i), cow

    def append_slots(self, seq_ids):
        """One append per listed sequence in order, all or nothing: on OutOfBlocks
        (or an unknown sequence) the allocator is left as it was.  Unknown or swapped-out
        sequences are reported before any shortage of blocks."""
        if any(s not in self.tables or s in self.on_host for s in seq_ids):
            raise ValueError("unknown or swapped-out sequence")
        trial = copy.deepcopy(self)
        res = [trial.append_slot(s) for s in seq_ids]
        self.__dict__.update(trial.__dict__)
        return res

    def beam_step(self, beam_ids, parents, new_ids):
        """A beam-search step, all or nothing ([fullstackaihub] section 3, [initnode]
        section 3: beams share blocks by copy-on-write until one writes).  New beam j
        continues old beam parents[j]: it is forked from it, the old beams are freed in
        list order, the new beams take their ids, and each appends one token in order.
        Returns [(slot, (src, dst) or None)] per new beam."""
        beam_ids, new_ids = [int(b) for b in beam_ids], [int(b) for b in new_ids]
        parents = [int(p) for p in parents]
        if len(set(beam_ids)) != len(beam_ids) or any(b not in self.tables or b in self.on_host for b in beam_ids):
            raise ValueError("old beams unknown or repeated")
        if len(parents) != len(new_ids) or any(not 0 <= p < len(beam_ids) for p in parents):
            raise ValueError("bad parent index")
        if len(set(new_ids)) != len(new_ids) or any(b in self.tables and b not in beam_ids for b in new_ids):
            raise ValueError("new beam ids repeated or taken")
        trial = copy.deepcopy(self)
        temp = [("beam", j) for j in range(len(new_ids))]      # ids no caller can hold
        for j, p in enumerate(parents):
            trial.fork(beam_ids[p], temp[j])
        for b in beam_ids:
            trial.free_seq(b)
        for j, b in enumerate(new_ids):
            trial.tables[b] = trial.tables.pop(temp[j])
            trial.ntokens[b] = trial.ntokens.pop(temp[j])
        res = trial.append_slots(new_ids)
        self.__dict__.update(trial.__dict__)
        return res

    def free_seq(self, seq_id):
        if seq_id not in self.tables:
            raise ValueError("unknown sequence")
        if seq_id in self.on_host:
            self.host_free.extend(self.tables.pop(seq_id))
            self.on_host.discard(seq_id)
        else:
            for blk in self.tables.pop(seq_id):
                self._release(blk)
        del self.ntokens[seq_id]

    def add_host_pool(self, num_host_blocks):
        if num_host_blocks <= 0 or self.num_host_blocks:
            raise ValueError("bad host pool")
        self.num_host_blocks = num_host_blocks
        self.host_free = deque(range(num_host_blocks))

    def swap_out(self, seq_id):
        """Moves a resident sequence to host blocks; returns [(device, host)] in table order."""
        if seq_id not in self.tables or seq_id in self.on_host:
            raise ValueError("unknown or swapped-out sequence")
        table = self.tables[seq_id]
        if len(table) > len(self.host_free):
            raise OutOfBlocks()
        pairs = []
        for i, blk in enumerate(table):
            h = self.host_free.popleft()
            pairs.append((blk, h))
            self._release(blk)
            table[i] = h
        self.on_host.add(seq_id)
        return pairs

    def swap_in(self, seq_id):
        """Brings a swapped-out sequence back to device blocks; returns [(host, device)]."""
        if seq_id not in self.on_host:
            raise ValueError("sequence is not swapped out")
        table = self.tables[seq_id]
        if len(table) > self.available():
            raise OutOfBlocks()
        pairs = []
        for i, h in enumerate(table):
            blk = self._take()
            pairs.append((h, blk))
            self.host_free.append(h)
            table[i] = blk
        self.on_host.discard(seq_id)
        return pairs

    def block_table(self, seq_id):
        return list(self.tables[seq_id])

    def num_free(self):
        return len(self.free)

    def num_cached_free(self):
        return len(self.unreferenced)

    def waste_tokens(self, seq_id):
        """Unused slots in the sequence's table (only its last block can be partial)."""
        return len(self.tables[seq_id]) * self.B - self.ntokens[seq_id]
