"""Reference model of the host block manager (allocation, sharing, copy-on-write).

TEST INFRASTRUCTURE: only tests and the benchmark's CPU legs use it.

It restates the pages' description in the plainest form:
  * "Efficient Memory Management for Large Language Model Serving with
    PagedAttention" summary page (xasun.com article 3997), section 2: a
    KV-cache manager maps each sequence's logical blocks to physical blocks
    and allocates and reclaims them on demand; section 1 and 2: blocks are
    shared through reference counts and copied on write for parallel
    sampling, beam search and shared prefixes; the scheduler evicts
    all-or-nothing when memory runs out.
  * "PyTorch-CUDA-v2.9 image enables PagedAttention" page, workflow list:
    a global page pool is created up front; finished requests' pages go
    back to the pool at once.

Policy choices the pages leave open (ours, stated once):
  * free blocks are handed out first-in first-out from a list whose initial
    order the caller gives (default 0..num_blocks-1); freed blocks go to the
    tail;
  * a request that needs more blocks than are free fails and changes
    nothing (all-or-nothing);
  * appending into a shared, partially filled last block copies it first
    (source keeps its other owners); the owner that finds the count at one
    writes in place.
"""
from collections import deque


class OutOfBlocks(Exception):
    pass


class BlockManagerModel:
    def __init__(self, num_blocks, block_size, free_order=None):
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        assert sorted(order) == list(range(num_blocks))
        self.free = deque(order)
        self.ref = [0] * num_blocks
        self.fill = [0] * num_blocks     # token slots written in each physical block
        self.tables = {}                 # seq id -> list of physical block ids
        self.lens = {}                   # seq id -> number of tokens

    # -- helpers ---------------------------------------------------------
    def _take(self, n):
        if n > len(self.free):
            raise OutOfBlocks(n)
        out = [self.free.popleft() for _ in range(n)]
        for b in out:
            assert self.ref[b] == 0
            self.ref[b] = 1
            self.fill[b] = 0
        return out

    def _release(self, b):
        self.ref[b] -= 1
        assert self.ref[b] >= 0
        if self.ref[b] == 0:
            self.fill[b] = 0
            self.free.append(b)

    # -- operations --------------------------------------------------------
    def allocate(self, seq, num_tokens):
        """Blocks for a new sequence of num_tokens (prefill)."""
        assert seq not in self.tables
        need = -(-num_tokens // self.block_size)
        blocks = self._take(need)
        for j, b in enumerate(blocks):
            self.fill[b] = min(self.block_size, num_tokens - j * self.block_size)
        self.tables[seq] = blocks
        self.lens[seq] = num_tokens
        return list(blocks)

    def fork(self, parent, child):
        """Child shares every block of parent (reference count + 1 each)."""
        assert child not in self.tables
        self.tables[child] = list(self.tables[parent])
        self.lens[child] = self.lens[parent]
        for b in self.tables[child]:
            self.ref[b] += 1

    def append_slot(self, seq):
        """Slot for the sequence's next token; returns (slot, cow) with cow =
        (src, dst) when the shared last block had to be copied, else None."""
        table = self.tables[seq]
        t = self.lens[seq]
        off = t % self.block_size
        cow = None
        if off == 0:
            (b,) = self._take(1)
            table.append(b)
        else:
            b = table[-1]
            if self.ref[b] > 1:
                (nb,) = self._take(1)
                self.fill[nb] = self.fill[b]
                self._release(b)
                table[-1] = nb
                cow = (b, nb)
                b = nb
        self.fill[b] = max(self.fill[b], off + 1)
        self.lens[seq] = t + 1
        return b * self.block_size + off, cow

    def swap_out(self, seq, host):
        """Move the whole sequence to the host-pool manager `host`, all or
        nothing; returns the (device block, host block) copies to make.  The
        host copies are private to the sequence (sharing ends at a swap)."""
        table = self.tables[seq]
        if len(table) > len(host.free):
            raise OutOfBlocks(len(table))
        dst = host._take(len(table))
        for d, b in zip(dst, table):
            host.fill[d] = self.fill[b]
        host.tables[seq] = list(dst)
        host.lens[seq] = self.lens[seq]
        pairs = list(zip(table, dst))
        self.free_seq(seq)
        return pairs

    def swap_in(self, seq, host):
        """The reverse of swap_out: the sequence returns from `host`."""
        return host.swap_out(seq, self)

    def free_seq(self, seq):
        for b in self.tables.pop(seq):
            self._release(b)
        del self.lens[seq]

    # -- queries -------------------------------------------------------------
    def num_free(self):
        return len(self.free)

    def utilisation(self):
        """Written token slots / slots of all blocks in use."""
        used = [b for b in range(self.num_blocks) if self.ref[b] > 0]
        if not used:
            return 0.0
        return sum(self.fill[b] for b in used) / (len(used) * self.block_size)

    def check_invariants(self):
        """Raise AssertionError if the bookkeeping is inconsistent."""
        count = [0] * self.num_blocks
        for seq, table in self.tables.items():
            assert len(table) == -(-self.lens[seq] // self.block_size)
            for b in table:
                count[b] += 1
        assert count == self.ref
        free = set(self.free)
        assert len(free) == len(self.free)
        for b in range(self.num_blocks):
            assert (b in free) == (self.ref[b] == 0)
        assert len(self.free) + sum(1 for r in self.ref if r > 0) == self.num_blocks
