"""Pure-Python model of the paged KV block pool (TEST INFRASTRUCTURE ONLY).

It is a second, independent statement of the allocation policy that the
native allocator implements, kept deliberately naive (lists and dicts) so the
native state can be compared with it bit-exactly after every operation.

What the pages fix:

* "一文读懂vLLM的…PagedAttention" page, section "运行模式的根本转变": one global
  pool of physical blocks is created at start-up; afterwards blocks are only
  taken from and given back to it, on demand.
* "Paged KV" wiki page, section "实现原理 / 运行阶段": prefill takes physical
  blocks in order; decode writes each new token into the next slot of the
  current block and takes a new block when that one is full.
* "PagedAttention 动态内存分页" page, sections "块粒度与块表" and "动态块分配与
  回收": a new block is appended to the tail of the sequence's block table,
  lazily, and a finished sequence's blocks return to the pool at once;
  section "写时复制与内存共享": sequences may reference the same physical blocks
  and a block is copied only when a sequence needs to write into it.

Readings where the pages are silent:

* the free pool is a LIFO stack that starts as [NB-1, ..., 1, 0] (top last),
  so the first allocation returns block 0, then 1, ...; freed blocks are
  pushed in table order; a pool may instead start from a given order (a
  seeded permutation scatters sequences over the physical blocks);
* an operation that runs out of blocks changes nothing and reports OOM;
* on append, a shared (refcount > 1) current block is copied into a fresh
  block, the old block loses one reference and the table entry is replaced;
  the last holder (refcount 1) writes in place;
* slot = physical_block * block_size + offset.

Block swapping ("PagedAttention 动态内存分页" page, 动态块分配与回收: when GPU
memory runs short, a sequence's KV blocks are moved to CPU memory and
brought back when needed).  Readings:

* the host pool is a second LIFO stack of host block ids, made once
  (``set_host_blocks``), first allocation 0, 1, ...;
* swap-out moves one whole sequence: in table order each block takes a host
  block (pair (gpu, host)), then the GPU block loses this sequence's
  reference (returning to the GPU stack at zero, in table order); a block
  still shared with a resident sequence stays on the GPU for it, and the
  swapped sequence keeps its own host copy;
* swap-in is the reverse: each host block takes a GPU block (pair (host,
  gpu)) and returns to the host stack, in table order;
* either one that runs out of blocks changes nothing and reports OOM;
* a swapped-out sequence cannot be appended to or forked; freeing it
  returns its host blocks.
"""

OK = 0
ERR_INVALID = -1
ERR_OOM = -4


class PoolModel:
    def __init__(self, num_blocks, block_size, free_order=None):
        """``free_order``: optional initial order of the pool (a permutation
        of 0..NB-1; its first entry is taken first).  Default 0, 1, 2, ..."""
        if num_blocks < 0 or block_size <= 0:
            raise ValueError("bad pool shape")
        self.num_blocks = num_blocks
        self.block_size = block_size
        if free_order is None:
            free_order = range(num_blocks)
        free_order = [int(b) for b in free_order]
        if sorted(free_order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of the blocks")
        self.free = free_order[::-1]  # top of stack = end
        self.refcount = [0] * num_blocks
        self.tables = {}  # seq_id -> list of physical blocks
        self.tokens = {}  # seq_id -> number of tokens
        self.host_free = None  # host block stack, once set_host_blocks ran
        self.host_refcount = []
        self.swapped = set()  # sequences whose table lists host blocks

    # -- helpers ---------------------------------------------------------
    def _take(self):
        b = self.free.pop()
        self.refcount[b] = 1
        return b

    def blocks_needed(self, num_tokens):
        return -(-num_tokens // self.block_size)

    # -- operations ------------------------------------------------------
    def seq_add(self, seq_id, num_tokens):
        """Prefill: a new sequence of num_tokens tokens takes its blocks in
        order from the pool."""
        if seq_id in self.tables or num_tokens < 0:
            return ERR_INVALID
        need = self.blocks_needed(num_tokens)
        if need > len(self.free):
            return ERR_OOM
        self.tables[seq_id] = [self._take() for _ in range(need)]
        self.tokens[seq_id] = num_tokens
        return OK

    def seq_fork(self, parent, child):
        """The child shares every block of the parent (one more reference)."""
        if parent not in self.tables or child in self.tables or parent in self.swapped:
            return ERR_INVALID
        self.tables[child] = list(self.tables[parent])
        self.tokens[child] = self.tokens[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1
        return OK

    def seq_append(self, seq_id):
        """Reserve the slot of one new token.  Returns (status, slot, cow_src,
        cow_dst); cow_src/cow_dst are -1 when no copy is needed."""
        if seq_id not in self.tables or seq_id in self.swapped:
            return ERR_INVALID, -1, -1, -1
        table = self.tables[seq_id]
        off = self.tokens[seq_id] % self.block_size
        src = dst = -1
        if off == 0:
            if not self.free:
                return ERR_OOM, -1, -1, -1
            table.append(self._take())
        else:
            last = table[-1]
            if self.refcount[last] > 1:
                if not self.free:
                    return ERR_OOM, -1, -1, -1
                new = self._take()
                self.refcount[last] -= 1
                table[-1] = new
                src, dst = last, new
        self.tokens[seq_id] += 1
        return OK, table[-1] * self.block_size + off, src, dst

    def seq_free(self, seq_id):
        if seq_id not in self.tables:
            return ERR_INVALID
        if seq_id in self.swapped:
            self.swapped.discard(seq_id)
            for h in self.tables.pop(seq_id):
                self.host_refcount[h] -= 1
                if self.host_refcount[h] == 0:
                    self.host_free.append(h)
            del self.tokens[seq_id]
            return OK
        for b in self.tables.pop(seq_id):
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free.append(b)
        del self.tokens[seq_id]
        return OK

    # -- swapping ----------------------------------------------------------
    def set_host_blocks(self, num_host_blocks):
        """Make the host pool (once): host blocks 0 .. num_host_blocks-1."""
        if self.host_free is not None or num_host_blocks < 0:
            return ERR_INVALID
        self.host_free = list(range(num_host_blocks))[::-1]
        self.host_refcount = [0] * num_host_blocks
        return OK

    def seq_swap_out(self, seq_id):
        """Move a resident sequence to host blocks.  Returns (status,
        [(gpu_block, host_block), ...]) in table order."""
        if (self.host_free is None or seq_id not in self.tables
                or seq_id in self.swapped):
            return ERR_INVALID, []
        table = self.tables[seq_id]
        if len(table) > len(self.host_free):
            return ERR_OOM, []
        pairs = []
        for b in table:
            h = self.host_free.pop()
            self.host_refcount[h] = 1
            pairs.append((b, h))
        for b in table:
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free.append(b)
        self.tables[seq_id] = [h for _, h in pairs]
        self.swapped.add(seq_id)
        return OK, pairs

    def seq_swap_in(self, seq_id):
        """Bring a swapped-out sequence back to GPU blocks.  Returns (status,
        [(host_block, gpu_block), ...]) in table order."""
        if seq_id not in self.swapped:
            return ERR_INVALID, []
        table = self.tables[seq_id]
        if len(table) > len(self.free):
            return ERR_OOM, []
        pairs = [(h, self._take()) for h in table]
        for h in table:
            self.host_refcount[h] -= 1
            if self.host_refcount[h] == 0:
                self.host_free.append(h)
        self.tables[seq_id] = [g for _, g in pairs]
        self.swapped.discard(seq_id)
        return OK, pairs

    # -- observations ----------------------------------------------------
    def num_free(self):
        return len(self.free)

    def waste(self, seq_id):
        """Slots allocated to the sequence but not holding a token."""
        return len(self.tables[seq_id]) * self.block_size - self.tokens[seq_id]

    def state(self):
        """Everything the native allocator must agree with, bit for bit."""
        return (
            tuple(self.free),
            tuple(self.refcount),
            tuple(sorted((s, tuple(t), self.tokens[s]) for s, t in self.tables.items())),
        )

    def host_state(self):
        """The host pool and which sequences are swapped out."""
        return (tuple(self.host_free or ()), tuple(self.host_refcount),
                tuple(sorted(self.swapped)))
