"""Block arithmetic and the host block manager (oracle; test infrastructure only).

What the pages fix, restated:

* A sequence's KV is split into fixed-size blocks of ``B`` token slots.
  Logical block ``j`` holds positions ``[jB, (j+1)B)``; a per-sequence block
  table maps logical block -> physical block, and physical blocks may sit
  anywhere in the pool ([PU] "按 Block 分配", the two bullet definitions;
  [ITHOME] "PagedAttention 的核心想法").
* Reading position ``p`` means: logical block ``p // B``, look it up in the
  table, read slot ``p % B`` inside that physical block ([PU] "按 Block 分配",
  the worked example: table [3, 0, 4], position 8 -> logical 2 -> P4, slot 0).
* Length ``T`` occupies ``ceil(T/B)`` blocks and ``B*ceil(T/B)`` slots; only
  the tail block has empty slots, fewer than ``B`` ([PU] "按 Block 分配", the
  ceil formula and the 9-token / 3-block / 12-slot figure).
* A new token fills the tail block first and takes a free block only when the
  tail is full; a finished request drops its references and blocks with no
  users return to the pool ([ITHOME] "手動畫一次 block table":
  [7, 1] -> [7, 1, 3] with B = 4; [PU] "按 Block 分配").
* Sequences sharing a prompt point at the same physical blocks; a reference
  count tracks the users of each block; writing into a block whose count is
  above one first copies it, remaps the writer to the copy, then appends.
  Full prefix blocks stay shared ([PU] "共享前缀，分叉时 Copy-on-write" and
  its figure: A and B share [P3, P0] with 6 tokens, A copies P0 -> P4 and
  writes a, B keeps P0 and writes b, P3 stays shared).

Readings where the pages are silent:

* Positions are 0-based; the "8th token" of the [ITHOME] example is position 7.
* The order in which free blocks are handed out is an input (``free_order``);
  the pages pick "for example block 3".
* With more than two sharers, writers are served in the order they call
  ``append_slot``; each writer that sees a count above one copies, the last
  remaining user writes in place (this reproduces the [PU] A-copies /
  B-keeps example).
* Slots are numbered in the flat pool view ``physical_block * B + offset``.
"""

from collections import deque


def blocks_needed(num_tokens, block_size):
    """ceil(T / B): blocks a sequence of T tokens occupies ([PU] "按 Block 分配")."""
    if block_size <= 0:
        raise ValueError("block_size must be positive")
    if num_tokens < 0:
        raise ValueError("num_tokens must be >= 0")
    return -(-num_tokens // block_size)


def slots_occupied(num_tokens, block_size):
    """B * ceil(T / B): slots reserved by a sequence of T tokens."""
    return block_size * blocks_needed(num_tokens, block_size)


def translate(block_table, position, block_size):
    """Position -> (physical block, slot within the block).

    [PU] "按 Block 分配": find logical block ``position // B``, look it up in
    the block table, read slot ``position % B`` of that physical block.
    """
    logical = position // block_size
    if position < 0 or logical >= len(block_table):
        raise IndexError(f"position {position} outside the table")
    return int(block_table[logical]), position % block_size


def flat_slot(block_table, position, block_size):
    """Flat slot id ``physical * B + offset`` of a position."""
    phys, off = translate(block_table, position, block_size)
    return phys * block_size + off


class OutOfBlocks(RuntimeError):
    pass


class BlockManager:
    """Free list, per-sequence block tables, reference counts, copy-on-write.

    ``free_order`` fixes which free block is handed out next (first element
    first); blocks released later go to the back of the queue.
    """

    def __init__(self, num_blocks, block_size, free_order=None):
        if free_order is None:
            free_order = range(num_blocks)
        free_order = [int(b) for b in free_order]
        if sorted(free_order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.free = deque(free_order)
        self.refcount = [0] * num_blocks
        self.tables = {}
        self.lengths = {}
        self.copy_pairs = []  # (src, dst) recorded by copy-on-write, in order

    # -- allocation ---------------------------------------------------------
    def _take(self):
        if not self.free:
            raise OutOfBlocks("block pool exhausted")
        b = self.free.popleft()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def _drop(self, b):
        self.refcount[b] -= 1
        assert self.refcount[b] >= 0
        if self.refcount[b] == 0:
            self.free.append(b)

    def num_free(self):
        return len(self.free)

    def add_sequence(self, seq_id, num_tokens=0):
        """Register a sequence holding ``num_tokens`` cached tokens (prefill)."""
        if seq_id in self.tables:
            raise KeyError(f"sequence {seq_id} exists")
        n = blocks_needed(num_tokens, self.block_size)
        self.tables[seq_id] = [self._take() for _ in range(n)]
        self.lengths[seq_id] = num_tokens
        return list(self.tables[seq_id])

    def fork(self, parent, child):
        """Child shares every block of the parent; each count goes up by one."""
        if child in self.tables:
            raise KeyError(f"sequence {child} exists")
        table = list(self.tables[parent])
        for b in table:
            self.refcount[b] += 1
        self.tables[child] = table
        self.lengths[child] = self.lengths[parent]
        return list(table)

    def append_slot(self, seq_id):
        """Reserve the slot of the next token of ``seq_id`` and return it.

        Tail has room and is not shared -> write in place.  Tail has room but
        is shared -> copy-on-write: take a free block, record (tail, new) as a
        copy pair, remap the table, drop one reference on the old tail.  Tail
        full (or no blocks yet) -> take a free block.  Returns the flat slot id.
        """
        table = self.tables[seq_id]
        pos = self.lengths[seq_id]
        B = self.block_size
        if pos % B == 0:
            # every existing block is full (or none exists): new block, no copy
            assert len(table) == pos // B
            table.append(self._take())
        else:
            tail = table[-1]
            if self.refcount[tail] > 1:
                new = self._take()
                self.copy_pairs.append((tail, new))
                table[-1] = new
                self._drop(tail)
        self.lengths[seq_id] = pos + 1
        return flat_slot(table, pos, B)

    def free_sequence(self, seq_id):
        """Request finished: drop its references; unused blocks return to the pool."""
        for b in self.tables.pop(seq_id):
            self._drop(b)
        del self.lengths[seq_id]

    def take_copy_pairs(self):
        """Return and clear the copy pairs recorded since the last call."""
        pairs, self.copy_pairs = self.copy_pairs, []
        return pairs
