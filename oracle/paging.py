"""Paging bookkeeping of the oracle: page index, slots, free list, block tables (test infrastructure).

Sources (vLLM pages):
* "PagedAttention / Cache Engine" (dingiv.github.io/ai/compute/engine/vllm):
  the page of a position is ``position // block_size``; worked example: the
  100th token's KV lives in page 100 // 16 = 6.
* "PagedAttention / Block Manager" (same page): pages are handed out and taken
  back in O(1) with a free list (a bitmap is the other option named there).
* "vLLM 前世今生" section 3.2: blocks of 16 tokens, physical blocks need not be
  contiguous, the block table maps them, several sequences may point at one
  physical block (prefix sharing); blocks are allocated on demand and a
  finished sequence's blocks are freed.

Readings taken where the pages are silent:
* a slot is ``physical_block * block_size + position % block_size``;
* the free list is a stack: ``alloc`` pops the top, ``free`` of the last
  reference pushes the block back on top; it starts so that pops come out in
  a given order;
* a block shared by several sequences carries a reference count, and returns to
  the free list when the count falls to zero;
* unused block-table entries hold -1;
* with a shared prefix, each prefix block is allocated once, by the first
  sequence that reaches it, and every later sequence reaching it takes a
  reference to it;
* copy-on-write (前世今生 §3.2 names it for shared blocks): before a sequence writes into a block
  that other sequences also reference, it takes a fresh block, copies the page into it and moves
  its reference there.
"""
from __future__ import annotations

from typing import Iterable, List, Optional, Sequence

import numpy as np


def page_index(position: int, block_size: int = 16) -> int:
    """Logical page (block) of a token position."""
    return position // block_size


def slot_of(block_table_row: Sequence[int], position: int, block_size: int = 16) -> int:
    """Pool slot of ``position`` for one sequence: physical block * block_size + in-block offset."""
    return int(block_table_row[page_index(position, block_size)]) * block_size + position % block_size


class FreeListModel:
    """Plain free-list block manager with reference counts (a stack of free ids)."""

    def __init__(self, num_blocks: int, order: Optional[Iterable[int]] = None):
        order = list(range(num_blocks)) if order is None else [int(b) for b in order]
        assert sorted(order) == list(range(num_blocks)), "order must be a permutation of the pool"
        self.num_blocks = num_blocks
        self._stack: List[int] = list(reversed(order))  # top of stack = end of list
        self._ref = [0] * num_blocks

    def alloc(self) -> Optional[int]:
        if not self._stack:
            return None
        b = self._stack.pop()
        assert self._ref[b] == 0
        self._ref[b] = 1
        return b

    def incref(self, b: int) -> bool:
        if not (0 <= b < self.num_blocks) or self._ref[b] == 0:
            return False
        self._ref[b] += 1
        return True

    def free(self, b: int) -> bool:
        if not (0 <= b < self.num_blocks) or self._ref[b] == 0:
            return False
        self._ref[b] -= 1
        if self._ref[b] == 0:
            self._stack.append(b)
        return True

    def cow(self, b: int):
        """Copy-on-write of block b before a write: (block to write, whether its page must be copied).

        With one reference the block is written in place. Shared, the writer's reference moves to a
        fresh block (b loses one reference), whose page must first receive a copy of b's. None when
        b is not allocated or no block is free (nothing changes then).
        """
        if not (0 <= b < self.num_blocks) or self._ref[b] == 0:
            return None
        if self._ref[b] == 1:
            return b, False
        nb = self.alloc()
        if nb is None:
            return None
        self._ref[b] -= 1
        return nb, True

    def refcount(self, b: int) -> int:
        return self._ref[b] if 0 <= b < self.num_blocks else -1

    @property
    def num_free(self) -> int:
        return len(self._stack)


def build_block_tables(context_lens: Sequence[int], order: Sequence[int], num_blocks: int,
                       block_size: int = 16, shared_prefix_tokens: int = 0,
                       max_blocks: Optional[int] = None) -> np.ndarray:
    """Block tables [num_seqs, max_blocks] (int32, -1 padded) as a free list hands blocks out.

    Sequences are served in order; each takes ceil(ctx / block_size) blocks,
    one ``alloc`` per logical block. With a shared prefix (a whole number of
    blocks), prefix block j is allocated by the first sequence that reaches it
    and every later sequence reaching it points its entry j at it (``incref``).
    """
    lens = [int(c) for c in context_lens]
    assert shared_prefix_tokens % block_size == 0
    n_prefix = shared_prefix_tokens // block_size
    need = [-(-c // block_size) for c in lens]
    if max_blocks is None:
        max_blocks = max(1, max(need))
    fl = FreeListModel(num_blocks, order)
    bt = np.full((len(lens), max_blocks), -1, dtype=np.int32)
    prefix_blocks: List[int] = []
    for s, nb in enumerate(need):
        for j in range(nb):
            if j < n_prefix:
                if j == len(prefix_blocks):
                    b = fl.alloc()
                    assert b is not None, "pool exhausted"
                    prefix_blocks.append(b)
                else:
                    b = prefix_blocks[j]
                    assert fl.incref(b)
            else:
                b = fl.alloc()
                assert b is not None, "pool exhausted"
            bt[s, j] = b
    return bt


def slots_for_positions(block_tables: np.ndarray, seqs: Sequence[int], positions: Sequence[int],
                        block_size: int = 16) -> np.ndarray:
    """Slot of each (sequence, position) pair, int64."""
    return np.array([slot_of(block_tables[s], p, block_size) for s, p in zip(seqs, positions)], dtype=np.int64)


def utilization(token_counts: Sequence[int], block_size: int = 16, reserve_tokens: int = 0):
    """KV-memory utilisation of live sequences: tokens stored / token slots held.

    Paged (blocks on demand): sum n / sum block_size * ceil(n / block_size); at most block_size - 1
    slots per sequence are unused. Contiguous reservation of reserve_tokens per sequence (the
    pre-allocation the pages describe for earlier systems): sum n / (count * reserve_tokens).
    Source: "vLLM 前世今生" §3.1-3.2 and the notes page "PagedAttention" (pre-allocation waste and
    fragmentation vs fixed pages allocated on demand).
    """
    n = [int(x) for x in token_counts]
    total = sum(n)
    held = sum(block_size * (-(-x // block_size)) for x in n)
    paged = total / held if held else 1.0
    contiguous = total / (len(n) * reserve_tokens) if (n and reserve_tokens) else None
    return paged, contiguous
