"""Host-side block manager: free list, per-block reference counts, logical ->
physical block tables and copy-on-write decisions.

It produces the inputs of the device calls -- block tables, slot mappings and
the (src, dst) pairs of ``copy_blocks`` -- and performs no device work.

Behaviour, after "PagedAttention 与 Continuous Batching" (zwxr.cn):
  * section 3.1: the KV cache is cut into fixed-size blocks (16 tokens by
    default); a token takes a slot only once it is produced, and a finished
    request returns whole blocks;
  * section 3.2: each sequence owns a block table mapping logical block i to
    any free physical block; a new physical block is appended when the last
    one fills;
  * section 3.4: blocks are shared between sequences with reference counts;
    shared blocks are read-only and a sequence that is about to write into a
    shared block copies it first (copy-on-write).
The free list follows the allocator description of the intelliparadigm.com
page (section 3.1: a free-block list, reference counting).
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Dict, Iterable, List, Optional, Tuple


class OutOfBlocks(RuntimeError):
    pass


@dataclass
class _Seq:
    table: List[int] = field(default_factory=list)
    length: int = 0


class BlockManager:
    """Physical blocks [0, num_blocks); ``free_order`` fixes allocation order
    (a shuffled order scatters every sequence across the pool)."""

    def __init__(self, num_blocks: int, block_size: int,
                 free_order: Optional[Iterable[int]] = None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.num_blocks = num_blocks
        self.block_size = block_size
        order = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        if sorted(order) != list(range(num_blocks)):
            raise ValueError("free_order must be a permutation of range(num_blocks)")
        self._free: List[int] = order[::-1]          # pop() takes order[0] first
        self.refcount: List[int] = [0] * num_blocks
        self._seqs: Dict[int, _Seq] = {}
        self._next_id = 0

    # -- allocation -----------------------------------------------------------
    def _alloc_block(self) -> int:
        if not self._free:
            raise OutOfBlocks("no free physical block")
        b = self._free.pop()
        assert self.refcount[b] == 0
        self.refcount[b] = 1
        return b

    def _release_block(self, b: int) -> None:
        assert self.refcount[b] > 0
        self.refcount[b] -= 1
        if self.refcount[b] == 0:
            self._free.append(b)

    @property
    def num_free(self) -> int:
        return len(self._free)

    def add_sequence(self, num_tokens: int = 0) -> int:
        """A new sequence holding ``num_tokens`` tokens (e.g. a prefilled prompt)."""
        sid = self._next_id
        self._next_id += 1
        self._seqs[sid] = _Seq()
        for _ in range(num_tokens):
            self.append_slot(sid)
        return sid

    def fork(self, parent: int) -> int:
        """A child that shares every block of ``parent`` (reference count + 1)."""
        p = self._seqs[parent]
        sid = self._next_id
        self._next_id += 1
        self._seqs[sid] = _Seq(table=list(p.table), length=p.length)
        for b in p.table:
            self.refcount[b] += 1
        return sid

    def free(self, sid: int) -> None:
        s = self._seqs.pop(sid)
        for b in s.table:
            self._release_block(b)

    def append_slot(self, sid: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Reserve the slot of the sequence's next token.

        Returns ``(slot, cow)`` with ``slot = physical_block * block_size +
        offset`` and ``cow = (src, dst)`` when the target block was shared and
        had to be copied before the write, else ``None``.
        """
        s = self._seqs[sid]
        pos = s.length
        lb, off = divmod(pos, self.block_size)
        cow = None
        if lb == len(s.table):                      # the last block is full
            s.table.append(self._alloc_block())
        else:
            b = s.table[lb]
            if self.refcount[b] > 1:                # shared: copy before writing
                nb = self._alloc_block()
                self.refcount[b] -= 1
                s.table[lb] = nb
                cow = (b, nb)
        s.length = pos + 1
        return s.table[lb] * self.block_size + off, cow

    # -- views ------------------------------------------------------------------
    def block_table(self, sid: int) -> List[int]:
        return list(self._seqs[sid].table)

    def seq_len(self, sid: int) -> int:
        return self._seqs[sid].length

    def slot_of(self, sid: int, pos: int) -> int:
        """Physical slot of logical token ``pos`` (section 3.2 translation)."""
        s = self._seqs[sid]
        if not 0 <= pos < s.length:
            raise IndexError(pos)
        return s.table[pos // self.block_size] * self.block_size + pos % self.block_size

    def used_slots_waste(self) -> Tuple[int, int]:
        """(slots reserved in allocated blocks, slots holding tokens), counting
        shared blocks once -- the internal fragmentation left by paging."""
        held = {b for s in self._seqs.values() for b in s.table}
        tokens = 0
        seen = set()
        for s in self._seqs.values():
            for i, b in enumerate(s.table):
                if b in seen:
                    continue
                seen.add(b)
                tokens += min(self.block_size, s.length - i * self.block_size)
        return len(held) * self.block_size, tokens
