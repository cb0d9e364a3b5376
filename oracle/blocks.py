"""Block arithmetic and a reference block manager (oracle, test infrastructure).

Sources (page title, section):
  * "Paged Attention" (klaylearn.com glossary), definition: fixed-size blocks,
    a per-request block table from logical block to physical block, a pool of
    physical blocks; prefill allocates and fills blocks, decode appends into
    the tail block or triggers another allocation, finished requests return
    their blocks to the free list.
  * "PagedAttention — AI Glossary" (modelrefs.com), "How it works" steps 1-5:
    blocks are reference counted so sequences sharing a prefix point at the
    same physical blocks; copy-on-write copies only the block being written.
  * "What is paged attention in vLLM, and why does it matter?", Steps 1-4,
    "Worked example" and "Trade-offs and edge cases" (third point, sharing).

Plain Python over lists and dicts; nothing here is tuned.
"""

from __future__ import annotations


class OutOfBlocks(Exception):
    """The free pool cannot supply the blocks an operation needs."""


class InvalidBlockOp(Exception):
    """An id out of range, or a reference dropped from a free block."""


# ---------------------------------------------------------------- arithmetic

def blocks_for(num_tokens: int, block_size: int) -> int:
    """Blocks a sequence of `num_tokens` holds: the ceiling of tokens / block size.

    A new block is taken only when the last one is full ("What is paged
    attention in vLLM...", Step 4), so the count is ceil(n / block_size).
    """
    return -(-num_tokens // block_size)


def allocated_slots(num_tokens: int, block_size: int) -> int:
    """Token slots in the blocks a sequence holds (filled plus idle tail)."""
    return blocks_for(num_tokens, block_size) * block_size


def kv_bytes_per_token(num_layers: int, num_kv_heads: int, head_dim: int, elem_bytes: int) -> int:
    """Cache bytes one token costs: a K row and a V row per KV head per layer.

    "What is paged attention in vLLM...", Step 1: Llama 3 8B (32 layers, 8 KV
    heads, head size 128) costs 128 KiB per token.
    """
    return num_layers * num_kv_heads * head_dim * 2 * elem_bytes


def requests_that_fit(budget_bytes: float, bytes_per_request: float) -> int:
    """Whole requests of a given footprint that fit in a byte budget (floor)."""
    return int(budget_bytes // bytes_per_request)


def logical_position(t: int, block_size: int):
    """(logical block index, offset inside the block) of token position t.

    "Paged Attention" (klaylearn.com glossary), definition: the kernel computes
    the token's logical block and offset, then looks up the physical block.
    """
    return t // block_size, t % block_size


def slot_of(block_table, t: int, block_size: int) -> int:
    """Flat slot index of token t: physical block * block_size + offset."""
    logical_block, offset = logical_position(t, block_size)
    return int(block_table[logical_block]) * block_size + offset


# ------------------------------------------------------ reference block manager

class BlockManager:
    """Free list + per-block reference counts + per-sequence block tables.

    * Free list: a LIFO stack of physical block ids. `set_free_order(ids)` makes
      the next allocations return ids[0], ids[1], ... in that order.
    * `alloc()` pops a free block and gives it reference count 1.
    * `decref()` drops one reference; at zero the block goes back on the stack
      ("What is paged attention in vLLM...", Step 4: blocks return to a free
      pool when the request ends).
    * Sequences: a list of physical ids in token order (the block table) and a
      token count.
    * `append_slot(seq)`: a new block is taken only when the tail block is full;
      if the tail block is shared (count > 1) it is first copied into a fresh
      block, the sequence drops its reference to the shared one and writes into
      its own copy ("PagedAttention — AI Glossary", How it works, step 5).
    * `fork(seq)`: the child points at the parent's blocks, each count + 1
      ("PagedAttention — AI Glossary", How it works, step 4).
    """

    def __init__(self, num_blocks: int, block_size: int):
        if num_blocks <= 0 or block_size <= 0:
            raise InvalidBlockOp("pool and block size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        self.refcount = [0] * num_blocks
        # top of the stack is the END of the list; initial order pops 0, 1, 2, ...
        self.free = list(range(num_blocks - 1, -1, -1))
        self.tables = {}   # seq id -> list of physical block ids
        self.lengths = {}  # seq id -> tokens written
        self._next_seq = 0

    # -- pool ------------------------------------------------------------
    def num_free(self) -> int:
        return len(self.free)

    def set_free_order(self, ids) -> None:
        ids = [int(i) for i in ids]
        if sorted(ids) != sorted(self.free):
            raise InvalidBlockOp("free order must list exactly the free blocks")
        self.free = list(reversed(ids))

    def alloc(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free blocks")
        b = self.free.pop()
        self.refcount[b] = 1
        return b

    def incref(self, b: int) -> None:
        self._check(b)
        if self.refcount[b] == 0:
            raise InvalidBlockOp(f"block {b} is free")
        self.refcount[b] += 1

    def decref(self, b: int) -> None:
        self._check(b)
        if self.refcount[b] == 0:
            raise InvalidBlockOp(f"block {b} is already free")
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self.free.append(b)

    def _check(self, b: int) -> None:
        if not 0 <= b < self.num_blocks:
            raise InvalidBlockOp(f"block id {b} out of range")

    # -- sequences -------------------------------------------------------
    def new_sequence(self) -> int:
        s = self._next_seq
        self._next_seq += 1
        self.tables[s] = []
        self.lengths[s] = 0
        return s

    def append_slot(self, s: int):
        """Reserve the slot of sequence s's next token.

        Returns (slot, cow) where cow is None or the (src, dst) block pair that
        must be copied before the token is written. On OutOfBlocks nothing
        changes.
        """
        table = self.tables[s]
        n = self.lengths[s]
        logical_block, offset = logical_position(n, self.block_size)
        cow = None
        if offset == 0:
            # tail full (or no block yet): take a new block
            table.append(self.alloc())
        else:
            tail = table[logical_block]
            if self.refcount[tail] > 1:
                fresh = self.alloc()
                self.decref(tail)
                table[logical_block] = fresh
                cow = (tail, fresh)
        self.lengths[s] = n + 1
        return slot_of(table, n, self.block_size), cow

    def add_tokens(self, s: int, count: int):
        """append_slot `count` times; returns (slots, cow pairs in order)."""
        need = self.blocks_needed(s, count)
        if need > len(self.free):
            raise OutOfBlocks(f"need {need} blocks, {len(self.free)} free")
        slots, cows = [], []
        for _ in range(count):
            slot, cow = self.append_slot(s)
            slots.append(slot)
            if cow is not None:
                cows.append(cow)
        return slots, cows

    def blocks_needed(self, s: int, count: int) -> int:
        """Fresh blocks that `count` more tokens of sequence s will take."""
        n = self.lengths[s]
        table = self.tables[s]
        extra = blocks_for(n + count, self.block_size) - blocks_for(n, self.block_size)
        offset = n % self.block_size
        if count > 0 and offset != 0 and self.refcount[table[n // self.block_size]] > 1:
            extra += 1   # the shared tail is copied before the first write
        return extra

    def fork(self, s: int) -> int:
        child = self.new_sequence()
        for b in self.tables[s]:
            self.incref(b)
        self.tables[child] = list(self.tables[s])
        self.lengths[child] = self.lengths[s]
        return child

    def free_sequence(self, s: int) -> None:
        for b in self.tables.pop(s):
            self.decref(b)
        del self.lengths[s]
