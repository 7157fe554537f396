"""Seeded paged-attention problems for the tests (CPU, numpy bf16 bit arrays).

Built from ``paged_kv_attention_35_b200.synth`` draws only.  The pool is
filled block by block from each sequence's logical K/V rows (logical block
``j`` of sequence ``i`` is copied into physical block ``block_tables[i][j]``),
and every pool row that no sequence owns is poisoned with NaN, the way a
reused, never-cleared pool can hold anything.
"""

from __future__ import annotations

import numpy as np
import torch

from paged_kv_attention_35_b200 import synth


def to_bits(t: torch.Tensor) -> np.ndarray:
    return t.contiguous().view(torch.int16).numpy().view(np.uint16).copy()


def from_bits(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)


def assign_blocks(lens, bs, num_blocks, seed):
    """Hand out blocks of a seeded permutation in order; returns a -1 padded table."""
    order = synth.permutation(num_blocks, seed).tolist()
    need = [-(-int(L) // bs) for L in lens]
    if sum(need) > num_blocks:
        raise ValueError("pool too small")
    width = max(max(need), 1)
    bt = np.full((len(lens), width), -1, dtype=np.int32)
    k = 0
    for i, n in enumerate(need):
        bt[i, :n] = order[k:k + n]
        k += n
    return bt


def build_pool(logical, bt, bs, num_blocks, hkv, d, poison=True):
    """Pool bits [NB, bs, Hkv, D] holding each sequence's logical rows."""
    fill = synth.NAN_BF16_BITS if poison else 0
    pool = np.full((num_blocks, bs, hkv, d), fill, dtype=np.uint16)
    for i, rows in enumerate(logical):
        L = rows.shape[0]
        for j in range(-(-L // bs)):
            chunk = rows[j * bs:(j + 1) * bs]
            pool[bt[i, j], :chunk.shape[0]] = chunk
    return pool


def decode_problem(lens, hq, hkv, d, bs, num_blocks=None, seed=0, poison=True):
    lens = [int(L) for L in lens]
    need = sum(-(-L // bs) for L in lens)
    nb = num_blocks or max(need + 2, int(np.ceil(1.25 * need)))
    bt = assign_blocks(lens, bs, nb, seed + 7)
    q = to_bits(synth.bf16_normal((len(lens), hq, d), seed + 1))
    kl = [to_bits(synth.bf16_normal((L, hkv, d), seed + 100 + 2 * i)) for i, L in enumerate(lens)]
    vl = [to_bits(synth.bf16_normal((L, hkv, d), seed + 101 + 2 * i)) for i, L in enumerate(lens)]
    return dict(q=q, k_logical=kl, v_logical=vl, block_tables=bt, lens=np.asarray(lens, np.int32),
                k_pool=build_pool(kl, bt, bs, nb, hkv, d, poison),
                v_pool=build_pool(vl, bt, bs, nb, hkv, d, poison),
                num_blocks=nb, bs=bs, hq=hq, hkv=hkv, d=d)


def prefill_problem(q_lens, k_lens, hq, hkv, d, bs, num_blocks=None, seed=0, poison=True):
    q_lens = [int(x) for x in q_lens]
    k_lens = [int(x) for x in k_lens]
    need = sum(-(-L // bs) for L in k_lens)
    nb = num_blocks or max(need + 2, int(np.ceil(1.25 * need)))
    bt = assign_blocks(k_lens, bs, nb, seed + 7)
    q = to_bits(synth.bf16_normal((sum(q_lens), hq, d), seed + 1))
    kl = [to_bits(synth.bf16_normal((L, hkv, d), seed + 100 + 2 * i)) for i, L in enumerate(k_lens)]
    vl = [to_bits(synth.bf16_normal((L, hkv, d), seed + 101 + 2 * i)) for i, L in enumerate(k_lens)]
    cu_q = np.concatenate([[0], np.cumsum(q_lens)]).astype(np.int32)
    cu_k = np.concatenate([[0], np.cumsum(k_lens)]).astype(np.int32)
    return dict(q=q, k_logical=kl, v_logical=vl, block_tables=bt, cu_q=cu_q, cu_k=cu_k,
                q_lens=q_lens, k_lens=k_lens,
                k_pool=build_pool(kl, bt, bs, nb, hkv, d, poison),
                v_pool=build_pool(vl, bt, bs, nb, hkv, d, poison),
                num_blocks=nb, bs=bs, hq=hq, hkv=hkv, d=d)
