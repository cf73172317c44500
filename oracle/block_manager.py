"""Oracle of the host block manager -- TEST INFRASTRUCTURE ONLY.

Only tests, the package's smoke check and the benchmark's CPU baseline may
import this module; the product's host library (the native block manager in
libpkv.so) must never call it.

A plain, slow model of the block bookkeeping that the pages describe, written
step by step for reading against them:

* "PagedAttention 与 Continuous Batching" (zwxr.cn), section 3.1: the cache is
  cut into fixed-size blocks; a token takes a slot when it is produced; a
  finished request gives back whole blocks.  Section 3.2: a per-sequence block
  table maps logical block i to any free physical block; a new block is taken
  when the last one is full.  Section 3.4: blocks are shared between
  sequences with reference counts; a sequence about to write into a shared
  block copies it first (copy-on-write).
* "vLLM 深度解析" (intelliparadigm.com), section 3.1: a free-block list,
  reference counting combined with LRU reclamation.
* "前缀缓存" (the section "4. 前缀缓存：相同的前半部分只需计算一次" of the
  article on vLLM's scheduler, chunked prefill and prefix caching): every
  FULL block gets a key = hash(previous block's key, this block's token ids,
  extra information); a request finds existing blocks by key and skips their
  prefill; a finished request's blocks are not erased but parked in a queue
  of "free but still holding content" blocks, entered from the request's
  tail so that the tail is evicted first, and evicted least-recently-used
  when space is needed; the hash is sha256.

Readings where the pages are silent:
  * key of block i = sha256(key_{i-1} || token ids as little-endian int32 ||
    extras), with key_{-1} = 32 zero bytes;
  * allocation takes a never-cached free block first (in the free-list
    order), and evicts the least recently parked cached block only when no
    such block is left;
  * a block that fills up while appending is entered into the cache under
    its key unless that key already names another block (the first one
    keeps it);
  * a forked child shares every block of its parent, cached or not.
"""
from __future__ import annotations

import hashlib
from collections import OrderedDict
from typing import Dict, List, Optional, Sequence, Tuple

ROOT_KEY = bytes(32)


def block_key(prev: bytes, tokens: Sequence[int], extras: bytes = b"") -> bytes:
    """sha256(prev key || int32 LE token ids || extras)."""
    h = hashlib.sha256()
    h.update(prev)
    for t in tokens:
        h.update(int(t).to_bytes(4, "little", signed=True))
    h.update(extras)
    return h.digest()


class OutOfBlocks(RuntimeError):
    pass


class OracleBlockManager:
    def __init__(self, num_blocks: int, block_size: int, free_order: Optional[Sequence[int]] = None,
                 prefix_cache: bool = True):
        self.bs = block_size
        self.num_blocks = num_blocks
        self.free: List[int] = list(range(num_blocks)) if free_order is None else [int(b) for b in free_order]
        self.ref = [0] * num_blocks
        self.key_of: Dict[int, bytes] = {}          # cached block -> its key
        self.block_of: Dict[bytes, int] = {}        # key -> cached block
        self.parked: "OrderedDict[int, None]" = OrderedDict()  # free cached blocks, LRU first
        self.prefix_cache = prefix_cache
        self.tables: Dict[int, List[int]] = {}
        self.tokens: Dict[int, List[int]] = {}
        self.extras: Dict[int, bytes] = {}
        self.next_id = 0
        self.hits = 0        # blocks found in the cache
        self.evictions = 0

    # -- blocks --------------------------------------------------------------
    def _take(self) -> int:
        if self.free:
            b = self.free.pop(0)
        elif self.parked:
            b, _ = self.parked.popitem(last=False)   # least recently parked
            del self.block_of[self.key_of.pop(b)]
            self.evictions += 1
        else:
            raise OutOfBlocks("no free block")
        self.ref[b] = 1
        return b

    def _drop(self, b: int) -> None:
        self.ref[b] -= 1
        if self.ref[b] == 0:
            if b in self.key_of:
                self.parked[b] = None                # keeps its content and key
            else:
                self.free.append(b)

    def _keys(self, sid: int, upto_block: int) -> List[bytes]:
        keys, prev = [], ROOT_KEY
        toks = self.tokens[sid]
        for i in range(upto_block):
            prev = block_key(prev, toks[i * self.bs:(i + 1) * self.bs], self.extras[sid])
            keys.append(prev)
        return keys

    # -- sequences -------------------------------------------------------------
    def add_sequence(self, tokens: Sequence[int], extras: bytes = b"") -> Tuple[int, int]:
        """A prompt of len(tokens) tokens.  Returns (sequence id, number of
        leading tokens whose KV is already cached)."""
        n = len(tokens)
        nblk = (n + self.bs - 1) // self.bs
        full = n // self.bs
        keys, prev = [], ROOT_KEY
        if self.prefix_cache:
            for i in range(full):
                prev = block_key(prev, tokens[i * self.bs:(i + 1) * self.bs], bytes(extras))
                keys.append(prev)
        # the leading run of blocks already cached under this prompt's keys
        hit = 0
        while hit < len(keys) and keys[hit] in self.block_of:
            hit += 1
        # all or nothing: a parked hit leaves the pool too
        parked_hits = sum(1 for i in range(hit) if self.ref[self.block_of[keys[i]]] == 0)
        if nblk - hit > len(self.free) + len(self.parked) - parked_hits:
            raise OutOfBlocks("not enough free blocks for the prompt")
        sid = self.next_id
        self.next_id += 1
        self.tokens[sid] = [int(t) for t in tokens]
        self.extras[sid] = bytes(extras)
        table: List[int] = []
        self.tables[sid] = table
        for i in range(nblk):
            if i < hit:
                b = self.block_of[keys[i]]
                if self.ref[b] == 0:
                    del self.parked[b]
                self.ref[b] += 1
                self.hits += 1
            else:
                b = self._take()
                if self.prefix_cache and i < full and keys[i] not in self.block_of:
                    self.block_of[keys[i]] = b
                    self.key_of[b] = keys[i]
            table.append(b)
        return sid, hit * self.bs

    def fork(self, parent: int) -> int:
        sid = self.next_id
        self.next_id += 1
        self.tables[sid] = list(self.tables[parent])
        self.tokens[sid] = list(self.tokens[parent])
        self.extras[sid] = self.extras[parent]
        for b in self.tables[sid]:
            self.ref[b] += 1
        return sid

    def append_token(self, sid: int, token: int) -> Tuple[int, Optional[Tuple[int, int]]]:
        """Slot of the new token and the copy-on-write pair, if any."""
        table, toks = self.tables[sid], self.tokens[sid]
        pos = len(toks)
        lb, off = divmod(pos, self.bs)
        cow = None
        if lb == len(table):
            table.append(self._take())
        elif self.ref[table[lb]] > 1:
            src = table[lb]
            dst = self._take()
            self.ref[src] -= 1
            table[lb] = dst
            cow = (src, dst)
        toks.append(int(token))
        if self.prefix_cache and off == self.bs - 1:   # the block just filled up
            key = self._keys(sid, lb + 1)[lb]
            b = table[lb]
            if key not in self.block_of and b not in self.key_of:
                self.block_of[key] = b
                self.key_of[b] = key
        return table[lb] * self.bs + off, cow

    def free_sequence(self, sid: int) -> None:
        table = self.tables.pop(sid)
        self.tokens.pop(sid)
        self.extras.pop(sid)
        for b in reversed(table):                    # the tail is parked first
            self._drop(b)

    # -- views -------------------------------------------------------------------
    def block_table(self, sid: int) -> List[int]:
        return list(self.tables[sid])

    def seq_len(self, sid: int) -> int:
        return len(self.tokens[sid])

    def num_free(self) -> int:
        return len(self.free) + len(self.parked)

    def waste(self) -> Tuple[int, int]:
        """(slots reserved by blocks in use, slots holding a token), each block
        in use counted once."""
        fill: Dict[int, int] = {}
        for sid, table in self.tables.items():
            n = len(self.tokens[sid])
            for i, b in enumerate(table):
                fill[b] = max(fill.get(b, 0), min(self.bs, n - i * self.bs))
        return len(fill) * self.bs, sum(fill.values())
