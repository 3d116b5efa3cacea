"""Host-side refcounted KV block allocator with copy-on-write.

This is the bookkeeping half of paged KV caching. It decides which physical
block each logical block of a sequence lives in and which blocks must be copied
before a write. It moves no KV data: the copies it returns are executed by the
``kv_block_copy`` kernel (or by the oracle's block copy on the CPU).

What it follows:

* page "PagedAttention Analysis" (ryotta.opik.net), section 2: blocks hold a
  fixed number B of tokens and are attached on demand. The waste per
  sequence is therefore at most the unfilled part of its last block (B-1
  tokens).
* page "PagedAttention 논문 쉽게 읽기" (iplexlaw.co.kr), section 2: a new
  token goes into the free slot of the last block, and a fresh block is taken
  and appended to the table only when that block is full. Section 3 says the
  same for sharing: a block is shared by reference, a write into a shared block
  copies it first, and blocks nobody references any more are reclaimed.
* page "추론 엔진에서의 메모리 가상화" (molayo1419.me), copy-on-write section.
  Two branches reference blocks #10 and #11 (refcount 2 each). A branch that
  writes into the partially filled shared block gets a new block (#45). The
  contents are copied, that branch's table entry is repointed, and the old
  block's refcount drops by one.
* page "PagedAttention Analysis" (ryotta.opik.net), section 6, for swapping.
  Beside the GPU block allocator sits a CPU one. A preempted sequence's blocks
  are copied to CPU blocks, all of the sequence's blocks together or none
  (all-or-nothing). The swap space never holds more blocks than the GPU pool
  has, which bounds it. The moves this returns are executed by the
  ``kv_block_swap`` kernel (or by the oracle's block swap).

Allocation only updates integer indices on the host. It never touches device
memory, which matches the pages' point that block management needs no
``cudaMalloc`` during generation.
"""

from __future__ import annotations

import hashlib
from collections import Counter
from dataclasses import dataclass, field
from typing import List, Optional, Sequence, Tuple

import numpy as np


@dataclass(frozen=True)
class CowCopy:
    """One whole-block copy ``src -> dst`` that must run before a write."""

    src: int
    dst: int


@dataclass(frozen=True)
class BlockMove:
    """One whole-block copy from block ``src`` of one pool to block ``dst`` of another."""

    src: int
    dst: int


@dataclass
class SeqState:
    """A sequence's block table (logical -> physical) and its token count.

    ``on_host`` tells which pool the table's ids refer to: the GPU pool, or the
    swap space after the sequence was swapped out."""

    table: List[int] = field(default_factory=list)
    num_tokens: int = 0
    on_host: bool = False


class BlockAllocator:
    """Free list plus a refcount per physical block.

    ``free_order`` fixes the order in which free blocks are handed out. A
    seeded permutation of ``range(num_blocks)`` scatters sequences over the
    pool, and an explicit list reproduces a worked example.
    """

    def __init__(self, num_blocks: int, block_size: int,
                 free_order: Optional[Sequence[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        listed = set(order)
        if len(listed) != len(order) or any(b < 0 or b >= num_blocks for b in order):
            raise ValueError("free_order must list distinct block ids in [0, num_blocks)")
        # pop() takes from the end, so store the order reversed
        self._free: List[int] = order[::-1]
        self._ref = np.zeros(num_blocks, dtype=np.int64)
        for b in range(num_blocks):
            if b not in listed:
                self._ref[b] = 1 << 40  # never handed out
        self.copies: List[CowCopy] = []

    # -- primitive operations -------------------------------------------------
    @property
    def num_free(self) -> int:
        return len(self._free)

    def refcount(self, block: int) -> int:
        return int(self._ref[block])

    def allocate(self) -> int:
        if not self._free:
            raise MemoryError("KV block pool exhausted")
        b = self._free.pop()
        assert self._ref[b] == 0
        self._ref[b] = 1
        return b

    def free(self, block: int, reuse_last: bool = False) -> None:
        """Drop one reference. A block nobody references goes back to the free
        list: next in line to be handed out, or with ``reuse_last`` at the back
        of the line (a cached block that should survive as long as possible)."""
        if self._ref[block] <= 0:
            raise ValueError(f"block {block} freed more often than referenced")
        self._ref[block] -= 1
        if self._ref[block] == 0:
            if reuse_last:
                self._free.insert(0, block)
            else:
                self._free.append(block)

    def reference(self, block: int) -> None:
        """Add a reference to a block, taking it off the free list if it was free."""
        if self._ref[block] == 0:
            self._free.remove(block)
        self._ref[block] += 1

    # -- sequence-level operations -------------------------------------------
    def adopt(self, table: Sequence[int], num_tokens: int) -> SeqState:
        """Take over an existing block table (one reference per entry)."""
        if -(-int(num_tokens) // self.block_size) != len(table):
            raise ValueError("table length does not match the token count")
        for b in table:
            self.reference(int(b))
        return SeqState(table=[int(b) for b in table], num_tokens=int(num_tokens))

    def new_sequence(self, num_tokens: int) -> SeqState:
        """Attach ceil(num_tokens / B) fresh blocks for a prompt."""
        seq = SeqState()
        nb = -(-int(num_tokens) // self.block_size)
        seq.table = [self.allocate() for _ in range(nb)]
        seq.num_tokens = int(num_tokens)
        return seq

    def fork(self, seq: SeqState) -> SeqState:
        """A new sequence that shares every block of ``seq`` by reference."""
        for b in seq.table:
            self._ref[b] += 1
        return SeqState(table=list(seq.table), num_tokens=seq.num_tokens)

    def append_slot(self, seq: SeqState) -> Tuple[int, Optional[CowCopy]]:
        """Reserve the slot for the sequence's next token.

        Returns ``(slot, copy)`` where ``slot = phys_block * B + offset`` and
        ``copy`` is the copy-on-write that must run first, or ``None``.
        """
        B = self.block_size
        off = seq.num_tokens % B
        cow = None
        if off == 0:
            seq.table.append(self.allocate())
        else:
            last = seq.table[-1]
            if self._ref[last] > 1:
                new = self.allocate()
                cow = CowCopy(src=last, dst=new)
                self._ref[last] -= 1
                seq.table[-1] = new
                self.copies.append(cow)
        slot = seq.table[-1] * B + off
        seq.num_tokens += 1
        return slot, cow

    def release(self, seq: SeqState) -> None:
        for b in seq.table:
            self.free(b)
        seq.table = []
        seq.num_tokens = 0

    @staticmethod
    def waste_slots(seq: SeqState, block_size: int) -> int:
        """Reserved but unfilled slots of a sequence (its last block only)."""
        return len(seq.table) * block_size - seq.num_tokens


class SwapSpace:
    """A CPU block allocator beside a GPU one, for swapping preempted sequences.

    ``swap_out`` moves every block of a group of sequences (for example the
    samples of one request, which may share blocks) into the swap space, and
    ``swap_in`` moves them back into the GPU pool. Both are all-or-nothing: if
    the target allocator cannot hold every distinct block of the group, nothing
    changes and MemoryError is raised. A block shared within the group moves
    once, and its refcount on the other side equals the number of table
    entries that reference it. The swap space is bounded by the GPU pool's
    block count.
    """

    def __init__(self, gpu: BlockAllocator, num_cpu_blocks: Optional[int] = None):
        n = gpu.num_blocks if num_cpu_blocks is None else int(num_cpu_blocks)
        if n > gpu.num_blocks:
            raise ValueError("the swap space holds at most as many blocks as the GPU pool")
        self.gpu = gpu
        self.cpu = BlockAllocator(n, gpu.block_size)

    def _move(self, seqs: Sequence[SeqState], src: BlockAllocator, dst: BlockAllocator,
              to_host: bool) -> List[BlockMove]:
        if any(sq.on_host == to_host for sq in seqs):
            raise ValueError("every sequence of the group must be on the source side")
        distinct: List[int] = []  # the group's source blocks, in first-use order
        seen = set()
        for sq in seqs:
            for b in sq.table:
                if b not in seen:
                    seen.add(b)
                    distinct.append(b)
        if len(distinct) > dst.num_free:
            raise MemoryError("not enough free blocks for the whole group")
        mapping = {b: dst.allocate() for b in distinct}  # one reference each
        for sq in seqs:
            old = sq.table
            sq.table = [mapping[b] for b in old]
            sq.on_host = to_host
            for b in old:  # the group's references leave the source side
                src.free(b)
        # one reference per table entry on the destination side
        counts = Counter(nb for sq in seqs for nb in sq.table)
        for nb, c in counts.items():
            for _ in range(c - 1):
                dst.reference(nb)
        return [BlockMove(src=b, dst=mapping[b]) for b in distinct]

    def swap_out(self, seqs: Sequence[SeqState]) -> List[BlockMove]:
        """GPU -> swap space. Returns the moves (GPU block -> CPU block). The
        moves must run before the freed GPU blocks are handed out again."""
        return self._move(seqs, self.gpu, self.cpu, True)

    def swap_in(self, seqs: Sequence[SeqState]) -> List[BlockMove]:
        """Swap space -> GPU. Returns the moves (CPU block -> GPU block)."""
        return self._move(seqs, self.cpu, self.gpu, False)


class BeamSearch:
    """The block bookkeeping of beam search for one request (page "PagedAttention
    Analysis", ryotta.opik.net, section 4: the beams share the prompt and
    intermediate blocks, and which blocks they share changes every step).

    Each ``step`` takes, for every new beam, the index of the surviving beam it
    continues. The new beams fork their parents (sharing every block by
    reference), the old beams are released, and each beam then takes the slot
    of its next token, copying its last block first when that block is shared.
    """

    def __init__(self, alloc: BlockAllocator, prompt_tokens: int, width: int):
        if width <= 0:
            raise ValueError("width must be positive")
        self.alloc = alloc
        root = alloc.new_sequence(prompt_tokens)
        self.beams: List[SeqState] = [root] + [alloc.fork(root) for _ in range(width - 1)]

    def step(self, parents: Sequence[int]) -> Tuple[List[int], List[CowCopy]]:
        """Returns the slots of the beams' next tokens and the block copies to
        run before those tokens are written."""
        if len(parents) != len(self.beams):
            raise ValueError("one parent per beam")
        new = [self.alloc.fork(self.beams[int(p)]) for p in parents]
        for b in self.beams:
            self.alloc.release(b)
        self.beams = new
        slots: List[int] = []
        copies: List[CowCopy] = []
        for b in self.beams:
            slot, cow = self.alloc.append_slot(b)
            slots.append(slot)
            if cow is not None:
                copies.append(cow)
        return slots, copies

    def blocks_in_use(self) -> int:
        return len({blk for b in self.beams for blk in b.table})

    def blocks_unshared(self) -> int:
        """Blocks the beams would hold without sharing (one table each)."""
        return sum(len(b.table) for b in self.beams)

    def release(self) -> None:
        for b in self.beams:
            self.alloc.release(b)
        self.beams = []


class PrefixCache:
    """Automatic prefix caching over a BlockAllocator (page "PagedAttention
    Analysis", ryotta.opik.net, section 4: each KV block is identified by a
    hash of the prefix tokens and registered in a global hash table, so common
    prefixes are shared without a tree).

    A full block's key is a hash of every token up to and including it (the
    previous block's key chained with this block's tokens): two sequences map a
    block to the same physical block exactly when their whole prefixes agree up
    to its end. A hit references the cached block; a miss allocates one, which
    the caller must fill, and registers it. A partial last block is always
    private and never cached. A released cached block keeps its contents and its
    key until the allocator hands it out again: it goes to the back of the free
    list, behind every block that holds nothing, and of one released prefix the
    later blocks go before the earlier ones.
    """

    def __init__(self, alloc: BlockAllocator):
        self.alloc = alloc
        self.table: dict = {}     # prefix key -> physical block
        self.key_of: dict = {}    # physical block -> prefix key
        self.hits = 0
        self.misses = 0

    @staticmethod
    def block_keys(tokens: Sequence[int], block_size: int) -> List[bytes]:
        keys, prev = [], b""
        for j in range(len(tokens) // block_size):
            blk = np.asarray(tokens[j * block_size:(j + 1) * block_size], dtype=np.int64)
            prev = hashlib.blake2b(prev + blk.tobytes(), digest_size=16).digest()
            keys.append(prev)
        return keys

    def _allocate(self) -> int:
        b = self.alloc.allocate()
        k = self.key_of.pop(b, None)
        if k is not None:  # evicted: its contents are about to be overwritten
            del self.table[k]
        return b

    def new_sequence(self, tokens: Sequence[int]) -> Tuple[SeqState, List[int]]:
        """The sequence's block table, and the logical blocks the caller must fill
        (the misses and the partial last block)."""
        B = self.alloc.block_size
        table, fills = [], []
        for j, k in enumerate(self.block_keys(tokens, B)):
            b = self.table.get(k)
            if b is not None:
                self.alloc.reference(b)
                self.hits += 1
            else:
                b = self._allocate()
                self.table[k] = b
                self.key_of[b] = k
                fills.append(j)
                self.misses += 1
            table.append(b)
        if len(tokens) % B:
            table.append(self._allocate())
            fills.append(len(table) - 1)
        return SeqState(table=table, num_tokens=len(tokens)), fills

    def release(self, seq: SeqState) -> None:
        # last block first: of a released prefix, the later blocks are evicted
        # before the earlier ones (a later key is useless without the earlier)
        for b in reversed(seq.table):
            self.alloc.free(b, reuse_last=b in self.key_of)
        seq.table = []
        seq.num_tokens = 0
