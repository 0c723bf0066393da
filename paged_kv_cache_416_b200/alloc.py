"""Host-side block allocator: free list plus per-block reference counts.

It only builds inputs for the device calls (block tables, slot mappings,
copy-on-write pairs); it owns no device memory and never calls the library.

Behaviour follows "PagedAttention" (Ultralytics glossary):

* §Sayfalama Nasıl Çalışır and its sketch: fixed-size blocks taken from a
  free list of scattered ids, popped from the head; a request needs
  ceil(len / block_size) blocks; a new block is taken only when the last one
  is full; token ``pos`` lives at (``table[pos // bs]``, ``pos % bs``).
* §Diziler Arasında Blokları Paylaşma: several block tables may name the same
  physical block, counted by a per-block reference count (parallel sampling,
  beam search, common prompts); before a sequence writes into a block that
  others still use, the block is copied (copy-on-write).
* §İlgili Teknikler, continuous batching: a finished sequence's blocks go back
  to the free pool at once.

Readings where the pages are silent: freed blocks are appended at the tail
of the free list; a write copies the block iff its reference count is above
one (the last holder writes in place).
"""

from __future__ import annotations

from collections import deque
from typing import Dict, Iterable, List, Optional, Tuple

import numpy as np


class OutOfBlocks(RuntimeError):
    """The free list is empty."""


class BlockAllocator:
    def __init__(self, num_blocks: int, block_size: int, free_list: Optional[Iterable[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = int(num_blocks)
        self.block_size = int(block_size)
        ids = list(range(self.num_blocks)) if free_list is None else [int(b) for b in free_list]
        if len(set(ids)) != len(ids) or any(b < 0 or b >= self.num_blocks for b in ids):
            raise ValueError("free list must hold distinct ids inside the pool")
        self.free: deque = deque(ids)
        self.refcount = np.zeros(self.num_blocks, dtype=np.int64)
        self.tables: Dict[int, List[int]] = {}
        self.lengths: Dict[int, int] = {}
        # prefix cache: chained block hash -> physical block holding that prefix
        self.cached: Dict[int, int] = {}
        self.block_hash: Dict[int, int] = {}

    # -- allocation ----------------------------------------------------------
    def _take(self) -> int:
        if not self.free:
            raise OutOfBlocks("no free block left in the pool")
        b = self.free.popleft()
        self.refcount[b] = 1
        return b

    def allocate(self, seq: int, num_tokens: int) -> List[int]:
        """Blocks for a new sequence of ``num_tokens`` tokens, taken from the
        head of the free list in order."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} already exists")
        n = -(-int(num_tokens) // self.block_size)
        self.tables[seq] = [self._take() for _ in range(n)]
        self.lengths[seq] = int(num_tokens)
        return list(self.tables[seq])

    def slot(self, seq: int, pos: int) -> int:
        """Slot id of token ``pos`` of ``seq``: physical block * bs + offset."""
        t = self.tables[seq]
        return t[pos // self.block_size] * self.block_size + pos % self.block_size

    def append_token(self, seq: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Grow ``seq`` by one token.  Returns the new token's slot and, when
        the write needs a copy-on-write, the (src, dst) block pair to copy
        before the write."""
        t = self.tables[seq]
        pos = self.lengths[seq]
        cow = None
        if pos % self.block_size == 0:
            t.append(self._take())  # the last block is full (or there is none)
        else:
            last = t[-1]
            if self.refcount[last] > 1:
                new = self._take()
                self.refcount[last] -= 1
                t[-1] = new
                cow = (last, new)
        self.lengths[seq] = pos + 1
        return self.slot(seq, pos), cow

    def fork(self, parent: int, child: int) -> None:
        """``child`` shares every block of ``parent`` (reference counts + 1)."""
        if child in self.tables:
            raise KeyError(f"sequence {child} already exists")
        self.tables[child] = list(self.tables[parent])
        self.lengths[child] = self.lengths[parent]
        for b in self.tables[child]:
            self.refcount[b] += 1

    def free_seq(self, seq: int) -> None:
        """Drop ``seq``; blocks nobody else uses return to the free list tail
        (and leave the prefix cache)."""
        for b in self.tables.pop(seq):
            self.refcount[b] -= 1
            if self.refcount[b] == 0:
                self.free.append(b)
                h = self.block_hash.pop(b, None)
                if h is not None and self.cached.get(h) == b:
                    del self.cached[h]
        del self.lengths[seq]

    # -- prefix cache ("PagedAttention", §Diziler Arasında Blokları Paylaşma:
    # hashing every block carries sharing across requests) -----------------
    def register_prefix(self, seq: int, hashes) -> None:
        """Remember the full blocks of ``seq`` under their chained hashes
        (``pa_hash_blocks`` of its tokens), so later requests with the same
        prefix can share them."""
        t = self.tables[seq]
        for j, h in enumerate(hashes):
            h = int(h) & ((1 << 64) - 1)
            if j >= len(t) or (j + 1) * self.block_size > self.lengths[seq]:
                break
            if h not in self.cached:
                self.cached[h] = t[j]
                self.block_hash[t[j]] = h

    def allocate_cached(self, seq: int, num_tokens: int, hashes) -> Tuple[List[int], int]:
        """Like :meth:`allocate`, but the leading full blocks whose chained
        hash is cached are shared (reference count + 1) instead of taken from
        the free list.  Returns (table, number of shared blocks)."""
        if seq in self.tables:
            raise KeyError(f"sequence {seq} already exists")
        n = -(-int(num_tokens) // self.block_size)
        table: List[int] = []
        for h in hashes:
            b = self.cached.get(int(h) & ((1 << 64) - 1))
            if b is None or len(table) >= n:
                break
            self.refcount[b] += 1
            table.append(b)
        shared = len(table)
        while len(table) < n:
            table.append(self._take())
        self.tables[seq] = table
        self.lengths[seq] = int(num_tokens)
        return list(table), shared

    # -- views ----------------------------------------------------------------
    def table_array(self, seqs: List[int], width: Optional[int] = None, pad: int = -1) -> np.ndarray:
        """int32 ``[len(seqs), width]`` block tables, padded with ``pad``."""
        w = max((len(self.tables[s]) for s in seqs), default=0) if width is None else int(width)
        out = np.full((len(seqs), max(w, 1)), pad, dtype=np.int32)
        for i, s in enumerate(seqs):
            t = self.tables[s]
            if len(t) > w:
                raise ValueError("table wider than requested width")
            out[i, : len(t)] = t
        return out

    def used_blocks(self) -> int:
        return int((self.refcount > 0).sum())
