"""Per-step metadata for the data plane (block tables, slots, lengths).

"Deep into the Nano-vLLM inference engine" (lnwmold.com), section
"Preparation before computation": a prefill batches several sequences and
computes their cumulative sequence lengths; a decode batches one new token
per sequence; both turn CPU-side token data into GPU tensors.  The slot of a
token at absolute position ``p`` of a sequence is row ``p % block_size`` of
physical block ``block_table[p // block_size]`` (block split rule, section
"From Sequences to Blocks").

All metadata is int32 (the kernels' index type); ``block_tables`` rows are
padded with -1.  Arrays are returned as numpy so the caller can place them in
pinned host memory and copy them to the device in one go.
"""

from __future__ import annotations

from dataclasses import dataclass

import numpy as np


@dataclass
class PrefillMetadata:
    cu_seqlens_q: np.ndarray        # [B+1] int32, new (computed) tokens per sequence
    cu_seqlens_k: np.ndarray        # [B+1] int32, all tokens per sequence
    max_seqlen_q: int
    max_seqlen_k: int
    slot_mapping: np.ndarray        # [total_q] int32, slot of every computed token
    positions: np.ndarray           # [total_q] int32, absolute position of every computed token
    block_tables: np.ndarray        # [B, max_blocks] int32, -1 padded

    @property
    def total_q(self) -> int:
        return int(self.cu_seqlens_q[-1])


@dataclass
class DecodeMetadata:
    slot_mapping: np.ndarray        # [B] int32, slot of each sequence's newest token
    context_lens: np.ndarray        # [B] int32, tokens to attend (newest included)
    block_tables: np.ndarray        # [B, max_blocks] int32, -1 padded
    max_context_len: int


def block_tables_array(seqs, min_width: int = 1) -> np.ndarray:
    width = max([min_width] + [len(s.block_table) for s in seqs])
    bt = np.full((len(seqs), width), -1, dtype=np.int32)
    for i, s in enumerate(seqs):
        bt[i, :len(s.block_table)] = s.block_table
    return bt


def slots_for(block_table, start: int, stop: int, block_size: int) -> np.ndarray:
    """Slots of absolute positions ``start .. stop-1`` of one sequence."""
    pos = np.arange(start, stop, dtype=np.int64)
    table = np.asarray(block_table, dtype=np.int64)
    return (table[pos // block_size] * block_size + pos % block_size).astype(np.int32)


def prepare_prefill(seqs, block_size: int) -> PrefillMetadata:
    cu_q = [0]
    cu_k = [0]
    slots, positions = [], []
    for s in seqs:
        n = len(s)
        start = s.num_cached_tokens
        if start >= n:
            raise ValueError(f"{s!r}: nothing to compute")
        cu_q.append(cu_q[-1] + n - start)
        cu_k.append(cu_k[-1] + n)
        slots.append(slots_for(s.block_table, start, n, block_size))
        positions.append(np.arange(start, n, dtype=np.int32))
    q_lens = np.diff(cu_q)
    k_lens = np.diff(cu_k)
    return PrefillMetadata(
        cu_seqlens_q=np.asarray(cu_q, dtype=np.int32),
        cu_seqlens_k=np.asarray(cu_k, dtype=np.int32),
        max_seqlen_q=int(q_lens.max()) if len(seqs) else 0,
        max_seqlen_k=int(k_lens.max()) if len(seqs) else 0,
        slot_mapping=np.concatenate(slots) if slots else np.zeros(0, np.int32),
        positions=np.concatenate(positions) if positions else np.zeros(0, np.int32),
        block_tables=block_tables_array(seqs),
    )


def prepare_decode(seqs, block_size: int) -> DecodeMetadata:
    slots = [0] * len(seqs)
    lens = [0] * len(seqs)
    for i, s in enumerate(seqs):
        n = len(s)
        pos = n - 1                      # the newest token
        slots[i] = s.block_table[pos // block_size] * block_size + pos % block_size
        lens[i] = n
    slots = np.asarray(slots, dtype=np.int32)
    lens = np.asarray(lens, dtype=np.int32)
    return DecodeMetadata(slot_mapping=slots, context_lens=lens,
                          block_tables=block_tables_array(seqs),
                          max_context_len=int(lens.max()) if len(seqs) else 0)
