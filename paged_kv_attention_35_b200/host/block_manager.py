"""BlockManager: the CPU control plane of the paged KV pool.

Sources
-------
* "Nano-vLLM engine architecture" (intelliparadigm.com), section 3.2
  "PagedAttention implementation": fixed-size blocks (default 256 tokens), a
  ``Block`` carries ``block_id``, ``ref_count`` and ``token_ids``; the manager
  keeps a deque of free blocks and a set of used ones and allocates from the
  left of the free deque; requests with equal prefixes share blocks by hash;
  blocks are allocated on demand as generation grows; sharing moves block ids,
  never data.
* "Deep into the Nano-vLLM inference engine" (lnwmold.com): section "From
  Sequences to Blocks" (fixed-size blocks, no block mixes two sequences, a
  long sequence spans many); section "Prefix Caching via hashing" (a
  hash -> block id map; a new sequence hashes its blocks, and a hit bumps the
  block's reference count and reuses it); section "Control plane vs. data
  plane" (the manager runs in CPU memory and only tracks metadata; freed
  blocks are marked free, their GPU memory is not cleared and is overwritten
  on reuse).

Readings where the pages are silent or disagree
-----------------------------------------------
* Fixed pool.  Page 2's ``allocate`` grows the pool when the free deque is
  empty; page 3 preempts when GPU memory is full.  The pool here is fixed and
  exhaustion is reported to the scheduler, which preempts.
* Free order.  The free deque starts as a seeded permutation of the block ids
  (a shuffled pool); allocation pops from the left, frees append on the right.
* Hash.  Only full blocks are hashed.  The hash is chained: block ``k``'s
  hash covers the previous block's hash and block ``k``'s token ids
  (blake2b, 8-byte digest, over the previous hash as 8 little-endian bytes and
  the ids as little-endian int32).  A hit also requires equal stored
  ``token_ids`` (collision guard).  After a sequence's first miss, its later
  blocks are not looked up.
* Freed blocks keep their hash entry while on the free list and can be
  revived by a hit; the entry is dropped when the block is handed out for
  other content.
* The block that holds a prompt's last token is never taken from the cache,
  so every prefill computes at least one query.
"""

from __future__ import annotations

import hashlib
from collections import deque

import numpy as np

from .sequence import Sequence


class Block:
    __slots__ = ("block_id", "ref_count", "hash", "token_ids")

    def __init__(self, block_id: int):
        self.block_id = block_id
        self.ref_count = 0
        self.hash = -1
        self.token_ids: list = []

    def __repr__(self) -> str:
        return f"Block({self.block_id}, ref={self.ref_count}, hash={self.hash:#x})"


def chain_hash(token_ids, prefix_hash: int = -1) -> int:
    """64-bit chained hash of one full block (see the module notes)."""
    h = hashlib.blake2b(digest_size=8)
    h.update(int(prefix_hash & 0xFFFFFFFFFFFFFFFF).to_bytes(8, "little"))
    h.update(np.asarray(token_ids, dtype="<i4").tobytes())
    return int.from_bytes(h.digest(), "little")


class PoolExhausted(RuntimeError):
    """No free block is left for a request that must make progress."""


class BlockManager:
    def __init__(self, num_blocks: int, block_size: int, seed=None):
        if num_blocks <= 0 or block_size <= 0:
            raise ValueError("num_blocks and block_size must be positive")
        self.block_size = int(block_size)
        self.num_blocks = int(num_blocks)
        self.blocks = [Block(i) for i in range(num_blocks)]
        if seed is None:
            order = range(num_blocks)
        else:
            order = np.random.default_rng(int(seed)).permutation(num_blocks).tolist()
        self.free_block_ids: deque = deque(int(b) for b in order)
        self.used_block_ids: set = set()
        self.hash_to_block_id: dict = {}
        # counters for reports
        self.prefix_hit_tokens = 0

    # ----------------------------------------------------------------- helpers
    @property
    def num_free_blocks(self) -> int:
        return len(self.free_block_ids)

    def _take_free_block(self, block_id=None) -> Block:
        """Hand out a free block (the leftmost one, or a named one being revived)."""
        if block_id is None:
            block_id = self.free_block_ids.popleft()
        else:
            self.free_block_ids.remove(block_id)
        blk = self.blocks[block_id]
        assert blk.ref_count == 0
        blk.ref_count = 1
        self.used_block_ids.add(block_id)
        return blk

    def _forget_hash(self, blk: Block) -> None:
        if blk.hash != -1 and self.hash_to_block_id.get(blk.hash) == blk.block_id:
            del self.hash_to_block_id[blk.hash]
        blk.hash = -1
        blk.token_ids = []

    def _register(self, blk: Block, h: int, token_ids) -> None:
        blk.hash = h
        blk.token_ids = list(token_ids)
        self.hash_to_block_id[h] = blk.block_id

    def _lookup(self, h: int, token_ids):
        bid = self.hash_to_block_id.get(h)
        if bid is None:
            return None
        blk = self.blocks[bid]
        return blk if blk.token_ids == list(token_ids) else None

    def _plan(self, seq: Sequence):
        """Walk a sequence's blocks: per block (tokens, hash or -1, cached block or None)."""
        bs = self.block_size
        n = len(seq)
        plan = []
        h = -1
        missed = False
        for i in range(seq.num_blocks(bs)):
            toks = seq.block_tokens(i, bs)
            full = len(toks) == bs
            h = chain_hash(toks, h) if full else -1
            hit = None
            # a full block that ends before the last token may come from the cache
            if full and not missed and (i + 1) * bs < n:
                hit = self._lookup(h, toks)
            if hit is None:
                missed = True
            plan.append((toks, h, hit))
        return plan

    # ------------------------------------------------------------- prefill side
    def blocks_needed(self, seq: Sequence) -> tuple:
        """(free blocks the allocation would take, tokens it would find cached)."""
        need = 0
        cached = 0
        for _, _, hit in self._plan(seq):
            if hit is None or hit.ref_count == 0:
                need += 1                      # fresh block, or a freed one revived
            if hit is not None:
                cached += self.block_size
        return need, cached

    def can_allocate(self, seq: Sequence) -> bool:
        return self.blocks_needed(seq)[0] <= len(self.free_block_ids)

    def allocate(self, seq: Sequence) -> None:
        """Give ``seq`` a block table covering all its tokens (prefix hits reused)."""
        if seq.block_table:
            raise ValueError("sequence already holds blocks")
        need, _ = self.blocks_needed(seq)
        if need > len(self.free_block_ids):
            raise PoolExhausted(f"need {need} blocks, {len(self.free_block_ids)} free")
        seq.num_cached_tokens = 0
        for toks, h, hit in self._plan(seq):
            if hit is not None:
                if hit.ref_count == 0:
                    self._take_free_block(hit.block_id)      # revive: contents still valid
                else:
                    hit.ref_count += 1
                seq.num_cached_tokens += self.block_size
                seq.block_table.append(hit.block_id)
                continue
            blk = self._take_free_block()
            self._forget_hash(blk)                          # old contents are dead now
            if h != -1:
                self._register(blk, h, toks)
            seq.block_table.append(blk.block_id)
        self.prefix_hit_tokens += seq.num_cached_tokens

    def deallocate(self, seq: Sequence) -> None:
        """Drop the sequence's references; blocks reaching zero go back to the free deque."""
        for bid in reversed(seq.block_table):
            blk = self.blocks[bid]
            blk.ref_count -= 1
            if blk.ref_count == 0:
                self.used_block_ids.discard(bid)
                self.free_block_ids.append(bid)             # contents kept, not zeroed
        seq.block_table = []
        seq.num_cached_tokens = 0

    # -------------------------------------------------------------- decode side
    def needs_new_block(self, seq: Sequence) -> bool:
        """Does the K/V row of the newest token (position len-1) start a new block?"""
        return len(seq.block_table) < seq.num_blocks(self.block_size)

    def can_append(self, seq: Sequence) -> bool:
        return (not self.needs_new_block(seq)) or len(self.free_block_ids) > 0

    def append_slot(self, seq: Sequence) -> None:
        """Make the block table cover the newest token; hash a block it completes."""
        bs = self.block_size
        if self.needs_new_block(seq):
            blk = self._take_free_block()
            self._forget_hash(blk)
            seq.block_table.append(blk.block_id)
        n = len(seq)
        if n % bs == 0:
            # the newest token fills its block: register the full block's hash
            last = n // bs - 1
            prev = self.blocks[seq.block_table[last - 1]].hash if last > 0 else -1
            toks = seq.block_tokens(last, bs)
            blk = self.blocks[seq.block_table[last]]
            if blk.ref_count == 1 and blk.hash == -1 and (last == 0 or prev != -1):
                self._register(blk, chain_hash(toks, prev), toks)

    # --------------------------------------------------------------- invariants
    def check_invariants(self, live_seqs) -> None:
        """Raise AssertionError if the pool bookkeeping is inconsistent."""
        refs = {}
        bs = self.block_size
        for s in live_seqs:
            # the table covers every computed token; the newest token may still lack its block
            lo = -(-(len(s) - 1) // bs)
            assert not s.block_table or lo <= len(s.block_table) <= s.num_blocks(bs), s
            for b in s.block_table:
                refs[b] = refs.get(b, 0) + 1
        for blk in self.blocks:
            assert blk.ref_count == refs.get(blk.block_id, 0), (blk, refs.get(blk.block_id))
            assert (blk.ref_count > 0) == (blk.block_id in self.used_block_ids)
        free = list(self.free_block_ids)
        assert len(free) == len(set(free))
        assert set(free).isdisjoint(self.used_block_ids)
        assert len(free) + len(self.used_block_ids) == self.num_blocks
        for h, bid in self.hash_to_block_id.items():
            assert self.blocks[bid].hash == h
