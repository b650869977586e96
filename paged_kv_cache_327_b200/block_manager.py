"""Host-side paged KV-cache bookkeeping: physical block pool and per-sequence block tables.

Follows the block-manager description on the vLLM pages:
  * "详解vLLM推理引擎架构" (tbr8.org), "PagedAttention 的核心思想": the cache is cut
    into fixed-size blocks (16 or 32 tokens); a block table maps each logical block of
    a sequence to a physical block anywhere in the pool (their example maps logical
    blocks 0, 1, 2 to physical pages 5, 12, 3).
  * same page, "Copy-on-Write 与内存共享": a fork shares every block of the parent and
    raises its refcount; a write to a block whose refcount exceeds 1 first allocates a
    new block, copies the old one into it, drops one reference from the old block and
    repoints the table entry.
  * "vLLM 深度解读" (luoboask.github.io), section 2 (BlockManager): a table needs
    ceil(num_tokens / block_size) blocks; the allocator hands out free physical ids and
    fails when none is left; append_slots adds one block when a sequence's last block
    is full.

Readings where the pages are silent or inconsistent:
  * the pages' allocator pops from an unordered set; here the free list is a seeded
    random permutation of range(num_blocks), popped from the front, which gives the
    shuffled physical placement the workloads need and keeps runs reproducible;
  * the pages' ``free`` ignores refcounts while ``fork_from`` raises them; here
    ``free`` drops one reference and returns the block to the pool at zero;
  * block copies are not executed on the host: ``copy_block`` records a (src, dst)
    pair that the device operation ``pa_copy_blocks`` carries out before the step's
    writes;
  * preemption ("详解vLLM推理引擎架构", scheduler section: a low-priority request's KV cache
    is moved to CPU memory and back): ``swap_out`` / ``swap_in`` move whole sequence groups
    between a GPU and a CPU allocator and return the block pairs for ``pa_swap_blocks``.
"""
from __future__ import annotations

import collections
from typing import Iterable, List, Optional, Tuple

import numpy as np


class NoFreeBlocksError(RuntimeError):
    """Raised when the physical block pool has no free block left."""


class BlockAllocator:
    """Pool of ``num_blocks`` physical KV blocks with reference counts.

    The free list is a permutation of ``range(num_blocks)`` drawn from ``seed`` (or
    the identity order when ``seed`` is None); ``allocate`` pops from its front.
    """

    def __init__(self, num_blocks: int, block_size: int, seed: Optional[int] = None,
                 rng: Optional[np.random.Generator] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        if rng is None and seed is not None:
            rng = np.random.default_rng(seed)
        order = rng.permutation(self.num_blocks) if rng is not None else np.arange(self.num_blocks)
        self._free = collections.deque(int(b) for b in order)
        self._refcount = np.zeros(self.num_blocks, dtype=np.int64)
        self._pending_copies: List[Tuple[int, int]] = []

    # -- allocation -------------------------------------------------------------------
    def allocate(self) -> int:
        if not self._free:
            raise NoFreeBlocksError(
                f"block pool exhausted: all {self.num_blocks} physical blocks are in use")
        block_id = self._free.popleft()
        self._refcount[block_id] = 1
        return block_id

    def free(self, block_id: int) -> None:
        """Drop one reference; the block returns to the pool when none is left."""
        self.decrement_refcount(block_id)
        if self._refcount[block_id] == 0:
            self._free.append(int(block_id))

    def get_num_free_blocks(self) -> int:
        return len(self._free)

    # -- reference counts -------------------------------------------------------------
    def _check(self, block_id: int) -> None:
        if not 0 <= block_id < self.num_blocks:
            raise IndexError(f"block id {block_id} outside the pool [0, {self.num_blocks})")

    def get_refcount(self, block_id: int) -> int:
        self._check(block_id)
        return int(self._refcount[block_id])

    def increment_refcount(self, block_id: int) -> None:
        self._check(block_id)
        if self._refcount[block_id] <= 0:
            raise ValueError(f"block {block_id} is not allocated")
        self._refcount[block_id] += 1

    def decrement_refcount(self, block_id: int) -> None:
        self._check(block_id)
        if self._refcount[block_id] <= 0:
            raise ValueError(f"refcount underflow on block {block_id}")
        self._refcount[block_id] -= 1

    # -- copy-on-write ------------------------------------------------------------------
    def copy_block(self, src: int, dst: int) -> None:
        """Record that physical block ``src`` must be duplicated into ``dst`` on the device."""
        self._check(src)
        self._check(dst)
        self._pending_copies.append((int(src), int(dst)))

    def take_pending_copies(self) -> np.ndarray:
        """Return the recorded (src, dst) pairs as int32 [P, 2] and clear the record."""
        pairs = np.asarray(self._pending_copies, dtype=np.int32).reshape(-1, 2)
        self._pending_copies = []
        return pairs


class BlockTable:
    """Logical-to-physical block map of one sequence."""

    def __init__(self, block_size: int = 16):
        self.block_size = int(block_size)
        self._blocks: List[int] = []
        self.num_tokens = 0

    def get_num_required_blocks(self, num_tokens: int) -> int:
        return -(-int(num_tokens) // self.block_size)

    def append_block(self, allocator: BlockAllocator) -> int:
        block_id = allocator.allocate()
        self._blocks.append(block_id)
        return block_id

    def fork_from(self, parent: "BlockTable", allocator: BlockAllocator) -> None:
        """Share every block of ``parent`` (copy-on-write)."""
        if parent.block_size != self.block_size:
            raise ValueError("block sizes differ")
        self._blocks = list(parent._blocks)
        self.num_tokens = parent.num_tokens
        for block_id in self._blocks:
            allocator.increment_refcount(block_id)

    def write_to_block(self, block_index: int, allocator: BlockAllocator) -> int:
        """Make logical block ``block_index`` private before a write; returns its physical id."""
        old = self._blocks[block_index]
        if allocator.get_refcount(old) > 1:
            new = allocator.allocate()
            allocator.copy_block(old, new)
            allocator.decrement_refcount(old)
            self._blocks[block_index] = new
        return self._blocks[block_index]

    def append_token(self, allocator: BlockAllocator) -> int:
        """Reserve the slot of the next token; returns slot = physical_block * block_size + offset.

        A full last block (or an empty table) gets a fresh block; a partial last block
        that is shared goes through copy-on-write first.
        """
        offset = self.num_tokens % self.block_size
        index = self.num_tokens // self.block_size
        if index >= len(self._blocks):
            self.append_block(allocator)
        phys = self.write_to_block(index, allocator)
        self.num_tokens += 1
        return phys * self.block_size + offset

    def append_tokens(self, n: int, allocator: BlockAllocator) -> np.ndarray:
        """Reserve slots for ``n`` tokens; same result as ``n`` calls of ``append_token``."""
        n = int(n)
        slots = np.empty(n, dtype=np.int64)
        done = 0
        while done < n:
            offset = self.num_tokens % self.block_size
            index = self.num_tokens // self.block_size
            if index >= len(self._blocks):
                self.append_block(allocator)
            phys = self.write_to_block(index, allocator)
            take = min(self.block_size - offset, n - done)
            slots[done:done + take] = phys * self.block_size + offset + np.arange(take)
            self.num_tokens += take
            done += take
        return slots

    def get_block_number(self, logical_block_idx: int) -> int:
        return self._blocks[logical_block_idx]

    def get_physical_blocks(self) -> List[int]:
        return list(self._blocks)

    def free(self, allocator: BlockAllocator) -> None:
        for block_id in self._blocks:
            allocator.free(block_id)
        self._blocks = []
        self.num_tokens = 0

    def __len__(self) -> int:
        return len(self._blocks)


def tables_to_array(tables: Iterable[BlockTable], max_blocks: Optional[int] = None,
                    pad: int = -1) -> np.ndarray:
    """Stack block tables into an int32 [N, max_blocks] array padded with ``pad``."""
    tables = list(tables)
    width = max([len(t) for t in tables] + [0]) if max_blocks is None else int(max_blocks)
    out = np.full((len(tables), max(width, 1)), pad, dtype=np.int32)
    for i, t in enumerate(tables):
        blocks = t.get_physical_blocks()
        if len(blocks) > out.shape[1]:
            raise ValueError("a table is wider than max_blocks")
        out[i, :len(blocks)] = blocks
    return out


def _move_tables(tables: Iterable[BlockTable], src: BlockAllocator, dst: BlockAllocator) -> np.ndarray:
    """Move every block the tables reference from pool ``src`` to pool ``dst``.

    A block shared by several of the tables moves once and stays shared (its new refcount is
    the number of references among the tables).  Returns the (src, dst) block pairs, in first-
    reference order, and repoints the tables to the new ids.
    """
    mapping = {}
    pairs = []
    for t in tables:
        for i, b in enumerate(t._blocks):
            if b in mapping:
                dst.increment_refcount(mapping[b])
            else:
                mapping[b] = dst.allocate()
                pairs.append((b, mapping[b]))
            t._blocks[i] = mapping[b]
            src.free(b)
    return np.asarray(pairs, dtype=np.int32).reshape(-1, 2)


def swap_out(tables: Iterable[BlockTable], gpu: BlockAllocator, cpu: BlockAllocator) -> np.ndarray:
    """Preempt a sequence group: its blocks move to the CPU pool (pairs gpu -> cpu)."""
    return _move_tables(tables, gpu, cpu)


def swap_in(tables: Iterable[BlockTable], cpu: BlockAllocator, gpu: BlockAllocator) -> np.ndarray:
    """Resume a swapped sequence group: its blocks move back to the GPU pool (pairs cpu -> gpu)."""
    return _move_tables(tables, cpu, gpu)


def find_prefix_groups(block_tables: np.ndarray, seq_lens: np.ndarray, block_size: int) -> np.ndarray:
    """Prefix groups for ``pa_decode_prefix``: runs of consecutive sequences whose tables start
    with the same physical blocks (forks of one parent, or requests that reuse one cached prompt:
    "详解vLLM推理引擎架构", "Copy-on-Write 与内存共享" and "Prefix Caching").

    Returns int32 [num_groups, 3] rows (first, members, shared): sequences first .. first +
    members - 1 (members >= 2) hold the same blocks for their first ``shared`` tokens, a
    positive multiple of block_size no larger than any member's length.  A block that is
    shared but only partly filled by some member is left out of ``shared`` (those tokens are
    read per sequence).
    """
    bt = np.asarray(block_tables)
    lens = np.asarray(seq_lens, dtype=np.int64)
    N = len(lens)
    rows = []
    i = 0
    while i < N:
        full_i = int(lens[i]) // block_size
        j = i + 1
        common = full_i
        while j < N and full_i > 0 and int(lens[j]) >= block_size and bt[j, 0] == bt[i, 0]:
            n = min(common, int(lens[j]) // block_size)
            same = bt[j, :n] == bt[i, :n]
            common = n if same.all() else int(np.argmin(same))
            j += 1
        if j - i >= 2 and common > 0:
            rows.append((i, j - i, common * block_size))
        i = j
    return np.asarray(rows, dtype=np.int32).reshape(-1, 3)
