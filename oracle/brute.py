"""Scalar pure-Python attention (``math.exp`` / ``math.fsum``) for tiny inputs.

TEST INFRASTRUCTURE ONLY.  A second formulation of the same definitions as
``oracle.paged``, written without numpy and without gathering: every key is
located through the block table one position at a time, and the causal rule
is stated as "key position <= query's absolute position".  It pins
``oracle.paged`` on tiny inputs (agreement to 1e-12).
"""

from __future__ import annotations

import math


def _row(pool, block_table, pos, head, block_size):
    blk = int(block_table[pos // block_size])
    return [float(x) for x in pool[blk][pos % block_size][head]]


def _attend(qvec, keys_vals, scale):
    scores = [scale * math.fsum(a * b for a, b in zip(qvec, k)) for k, _ in keys_vals]
    mx = max(scores)
    w = [math.exp(s - mx) for s in scores]
    z = math.fsum(w)
    d = len(keys_vals[0][1])
    return [math.fsum(w[t] * keys_vals[t][1][c] for t in range(len(w))) / z for c in range(d)]


def brute_decode(q, k_pool, v_pool, block_tables, context_lens, scale=None):
    """Decode attention; nested lists / arrays in, nested lists out."""
    B, hq, d = len(q), len(q[0]), len(q[0][0])
    bs = len(k_pool[0])
    hkv = len(k_pool[0][0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = []
    for i in range(B):
        rows = []
        for h in range(hq):
            g = (h * hkv) // hq          # == h // (hq // hkv) for integral groups
            kv = [(_row(k_pool, block_tables[i], t, g, bs), _row(v_pool, block_tables[i], t, g, bs))
                  for t in range(int(context_lens[i]))]
            rows.append(_attend([float(x) for x in q[i][h]], kv, scale))
        out.append(rows)
    return out


def brute_prefill(q, k_pool, v_pool, cu_seqlens_q, cu_seqlens_k, block_tables, scale=None):
    """Varlen causal prefill with cached prefix, one query at a time."""
    hq, d = len(q[0]), len(q[0][0])
    bs = len(k_pool[0])
    hkv = len(k_pool[0][0])
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    out = [None] * len(q)
    for i in range(len(cu_seqlens_q) - 1):
        q_start, q_end = int(cu_seqlens_q[i]), int(cu_seqlens_q[i + 1])
        k_len = int(cu_seqlens_k[i + 1]) - int(cu_seqlens_k[i])
        first_new_pos = k_len - (q_end - q_start)     # absolute position of query 0
        for r in range(q_start, q_end):
            qpos = first_new_pos + (r - q_start)
            rows = []
            for h in range(hq):
                g = (h * hkv) // hq
                kv = [(_row(k_pool, block_tables[i], t, g, bs), _row(v_pool, block_tables[i], t, g, bs))
                      for t in range(k_len) if t <= qpos]
                rows.append(_attend([float(x) for x in q[r][h]], kv, scale))
            out[r] = rows
    return out
