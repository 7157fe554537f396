"""numpy float64 oracle: store, gather, decode and varlen prefill attention.

TEST INFRASTRUCTURE ONLY (see the package docstring): the product path never
imports this module.

Sources and readings
--------------------
* Block pool and slots.  "Nano-vLLM engine architecture" (intelliparadigm.com),
  section 3.2 "PagedAttention implementation": GPU memory is cut into
  fixed-size blocks (default 256 tokens).  "Deep into the Nano-vLLM inference
  engine" (lnwmold.com), section "From Sequences to Blocks": a sequence is cut
  into fixed-size blocks, a long sequence spans many blocks, no block mixes two
  sequences.  The physical layout is deferred by the same page (section
  "What's Next"); reading taken: one K pool and one V pool per layer, each
  ``[num_blocks, block_size, num_kv_heads, head_dim]``, and a *slot* is the
  flat token row ``block_id * block_size + offset`` of the
  ``[num_blocks * block_size, num_kv_heads, head_dim]`` view.
* Store.  Each step's new K/V rows go to their slots; a negative slot means
  "no write" (padding reading).  The copy is exact: it moves bf16 bit
  patterns.
* Control plane vs data plane (lnwmold.com, section "Control plane vs. data
  plane"): freed blocks are not zeroed, so pool rows beyond a sequence's
  context hold stale data; the attention definitions below never read them.
* Attention.  Plain scaled-dot-product softmax attention over the gathered,
  contiguous K/V of each sequence, in float64, on the same bf16 inputs
  upcast exactly.  GQA reading: query head ``h`` uses KV head
  ``h // (Hq // Hkv)``.  Decode: one query per sequence attending to all of
  its ``context_len`` rows (the new token's row included, stored first).
  Prefill ("Model Runner", section "Preparation before computation":
  several sequences batched by cumulative sequence lengths): sequence ``i``
  brings ``q_len = cu_q[i+1]-cu_q[i]`` new queries and has
  ``k_len = cu_k[i+1]-cu_k[i]`` keys, the first ``k_len - q_len`` of them a
  cached prefix ("Prefix Caching via hashing"); query ``j`` sits at absolute
  position ``k_len - q_len + j`` and sees keys ``0 .. k_len - q_len + j``
  (bottom-right causal alignment).
"""

from __future__ import annotations

import math

import numpy as np


# ---------------------------------------------------------------------------
# bf16 <-> float64, by definition of the format (1 sign, 8 exponent, 7 stored
# mantissa bits; a bf16 value is the float32 with the same top 16 bits).
# ---------------------------------------------------------------------------

def bf16_bits_to_f64(bits: np.ndarray) -> np.ndarray:
    """Exact upcast of bf16 bit patterns (uint16 / int16 array) to float64."""
    b = np.asarray(bits).astype(np.uint16).astype(np.uint32) << np.uint32(16)
    with np.errstate(invalid="ignore"):
        return b.view(np.float32).astype(np.float64)


def f64_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float64 straight to bf16 (nearest, ties to even); returns uint16.

    Done in one rounding from float64 (no float32 intermediate, so no double
    rounding): a finite value is rounded to a multiple of its bf16 quantum
    ``2**(e - 8)`` where ``x = m * 2**e`` with ``0.5 <= |m| < 1``; exponents
    below the float32/bf16 normal range keep the subnormal quantum
    ``2**-133``.  Magnitudes that round to ``2**128`` or more become inf.
    """
    x = np.asarray(x, dtype=np.float64)
    out = np.empty(x.shape, dtype=np.float64)
    finite = np.isfinite(x)
    xf = x[finite]
    _, e = np.frexp(xf)
    e = np.maximum(e, -125)
    quantum = np.ldexp(1.0, e - 8)
    r = np.rint(xf / quantum) * quantum          # np.rint: ties to even
    r = np.where(np.abs(r) >= 2.0 ** 128, np.copysign(np.inf, r), r)
    out[finite] = r
    out[~finite] = x[~finite]
    f32 = out.astype(np.float32)                 # exact: r is representable
    bits = (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    nan = np.isnan(x)
    bits[nan] = np.uint16(0x7FC0)
    return bits


# ---------------------------------------------------------------------------
# a1 -- slot of a token position (block table lookup)
# ---------------------------------------------------------------------------

def ref_slot_mapping(block_table, positions, block_size: int) -> np.ndarray:
    """Slot of each absolute token position of one sequence.

    ``slot = block_table[pos // block_size] * block_size + pos % block_size``:
    the sequence's logical block ``pos // block_size`` lives in physical
    block ``block_table[...]`` (block split rule, lnwmold.com "From Sequences
    to Blocks"), at row ``pos % block_size`` of it.
    """
    out = []
    for pos in positions:
        out.append(int(block_table[pos // block_size]) * block_size + pos % block_size)
    return np.asarray(out, dtype=np.int64)


# ---------------------------------------------------------------------------
# a3 -- store_kvcache
# ---------------------------------------------------------------------------

def ref_store(k_pool_bits, v_pool_bits, key_bits, value_bits, slot_mapping):
    """Scatter new K/V rows into copies of the pools; returns (k_pool, v_pool).

    Pools are bf16 bit arrays ``[num_blocks, block_size, Hkv, D]``; key/value
    are ``[N, Hkv, D]``.  Row ``i`` goes to flat token row ``slot_mapping[i]``
    unless that slot is negative (skip).  Later rows win when two rows name
    the same slot (the order the rows are given in).
    """
    kp = np.array(k_pool_bits, copy=True)
    vp = np.array(v_pool_bits, copy=True)
    nb, bs, hkv, d = kp.shape
    kflat = kp.reshape(nb * bs, hkv, d)
    vflat = vp.reshape(nb * bs, hkv, d)
    for i, s in enumerate(np.asarray(slot_mapping).tolist()):
        if s < 0:
            continue
        kflat[s] = key_bits[i]
        vflat[s] = value_bits[i]
    return kp, vp


# ---------------------------------------------------------------------------
# gather -- the contiguous K (or V) of one sequence
# ---------------------------------------------------------------------------

def ref_gather(pool, block_table, length: int):
    """Rows ``0 .. length-1`` of one sequence, concatenated in logical order.

    ``pool``: ``[num_blocks, block_size, Hkv, D]`` (any dtype).  Physical
    block ``block_table[j]`` holds logical rows ``j*bs .. j*bs+bs-1``.
    Returns ``[length, Hkv, D]``.
    """
    bs = pool.shape[1]
    nblk = -(-length // bs)
    parts = [pool[int(block_table[j])] for j in range(nblk)]
    if not parts:
        return pool[:0, 0]
    return np.concatenate(parts, axis=0)[:length]


def _kv_head(h: int, group: int) -> int:
    """GQA reading: query heads ``g*group .. g*group+group-1`` share KV head ``g``."""
    return h // group


def _last_visible_key(k_len: int, q_len: int, j: int) -> int:
    """Bottom-right causal rule: query ``j`` sits at absolute position ``k_len-q_len+j``."""
    return (k_len - q_len) + j


def _default_scale(head_dim: int) -> float:
    return 1.0 / math.sqrt(head_dim)


def _softmax_attend(s, v):
    """``softmax(s) @ v`` for a 1-D score row (max-subtracted, float64)."""
    m = s.max()
    p = np.exp(s - m)
    return (p / p.sum()) @ v


# ---------------------------------------------------------------------------
# a4 -- paged decode attention
# ---------------------------------------------------------------------------

def ref_decode(q, k_pool, v_pool, block_tables, context_lens, scale=None):
    """Decode attention, float64.

    q: ``[B, Hq, D]`` float64 (bf16 values upcast); pools
    ``[NB, bs, Hkv, D]`` float64; ``block_tables [B, max_blocks]``;
    ``context_lens [B]`` (length after the new token was appended, so the
    new token's row -- stored before attention -- is attended).
    Returns ``[B, Hq, D]`` float64.
    """
    B, hq, d = q.shape
    hkv = k_pool.shape[2]
    group = hq // hkv
    if scale is None:
        scale = _default_scale(d)
    out = np.zeros((B, hq, d), dtype=np.float64)
    for i in range(B):
        L = int(context_lens[i])
        K = ref_gather(k_pool, block_tables[i], L)   # [L, Hkv, D]
        V = ref_gather(v_pool, block_tables[i], L)
        for h in range(hq):
            g = _kv_head(h, group)
            s = (K[:, g, :] @ q[i, h]) * scale
            out[i, h] = _softmax_attend(s, V[:, g, :])
    return out


# ---------------------------------------------------------------------------
# a5 -- varlen causal prefill with cached prefix
# ---------------------------------------------------------------------------

def ref_prefill(q, k_pool, v_pool, cu_seqlens_q, cu_seqlens_k, block_tables,
                scale=None):
    """Varlen causal prefill over paged KV, float64.

    q: ``[total_q, Hq, D]`` float64 packed by ``cu_seqlens_q``; keys of
    sequence ``i`` are its first ``k_len = cu_k[i+1]-cu_k[i]`` pool rows via
    ``block_tables[i]``.  Query ``j`` of sequence ``i`` (``q_len`` queries)
    attends keys ``t <= (k_len - q_len) + j``.
    Returns ``[total_q, Hq, D]`` float64.
    """
    total_q, hq, d = q.shape
    hkv = k_pool.shape[2]
    group = hq // hkv
    if scale is None:
        scale = _default_scale(d)
    out = np.zeros((total_q, hq, d), dtype=np.float64)
    nseq = len(cu_seqlens_q) - 1
    for i in range(nseq):
        q0, q1 = int(cu_seqlens_q[i]), int(cu_seqlens_q[i + 1])
        k_len = int(cu_seqlens_k[i + 1]) - int(cu_seqlens_k[i])
        q_len = q1 - q0
        if q_len == 0:
            continue
        K = ref_gather(k_pool, block_tables[i], k_len)
        V = ref_gather(v_pool, block_tables[i], k_len)
        for h in range(hq):
            g = _kv_head(h, group)
            S = (q[q0:q1, h, :] @ K[:, g, :].T) * scale          # [q_len, k_len]
            for j in range(q_len):
                last = _last_visible_key(k_len, q_len, j)
                out[q0 + j, h] = _softmax_attend(S[j, :last + 1], V[:last + 1, g, :])
    return out


def ref_prefill_flops(cu_seqlens_q, cu_seqlens_k, num_q_heads: int, head_dim: int) -> int:
    """Algorithmic FLOPs of a causal prefill: 4*D*Hq per visible (query, key) pair.

    Counted pair by pair (QK^T and PV each 2*D flops per pair), masked pairs
    excluded; used to pin the closed-form count the bench reports.
    """
    pairs = 0
    for i in range(len(cu_seqlens_q) - 1):
        q_len = int(cu_seqlens_q[i + 1]) - int(cu_seqlens_q[i])
        k_len = int(cu_seqlens_k[i + 1]) - int(cu_seqlens_k[i])
        cached = k_len - q_len
        for j in range(q_len):
            pairs += cached + j + 1
    return 4 * head_dim * num_q_heads * pairs
