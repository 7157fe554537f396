"""Synthetic workloads driven through the control plane and the C-ABI kernels.

Each workload places its sequences with the product's ``BlockManager`` (seeded,
shuffled free-block order), draws its K/V/q values from ``synth`` on the CPU,
and knows how to upload itself and run one step of the hot path on the GPU.
The logical (per-sequence, contiguous) K/V draws are kept on the host so a
checker can recompute the step from them independently.

* ``DecodeWorkload``        one decode step: the batch's prompt rows are
  stored in an untimed set-up; a step stores each sequence's newest K/V row
  (``store_kvcache``) and runs ``decode``.
* ``PrefixPrefillWorkload`` one prefill step with a prefix cache: a warm-up
  sequence's prefix is stored in an earlier (untimed) step, the batch is
  allocated through the hash prefix cache (shared prefix blocks are hits), a
  step stores the uncached rows and runs ``prefill_varlen``.
"""

from __future__ import annotations

import math

import numpy as np
import torch

from . import synth
from .host import BlockManager, Sequence, prepare_prefill, slots_for


def _nan_pool(shape, device):
    return torch.full(shape, synth.NAN_BF16_BITS, dtype=torch.int16, device=device).view(torch.bfloat16)


class DecodeWorkload:
    def __init__(self, lens, hq, hkv, d, bs, num_blocks=None, seed=0, pool_seed=None,
                 pool_factor=1.25):
        self.lens = [int(L) for L in lens]
        self.B = len(self.lens)
        self.hq, self.hkv, self.d, self.bs = hq, hkv, d, bs
        need = sum(-(-L // bs) for L in self.lens)
        self.nb = num_blocks or max(need + 1, int(math.ceil(pool_factor * need)))
        bm = BlockManager(self.nb, bs, seed=seed if pool_seed is None else pool_seed)
        self.seqs = [Sequence(synth.token_ids(L, seed * 7919 + i)) for i, L in enumerate(self.lens)]
        for s in self.seqs:
            bm.allocate(s)
        self.block_tables = np.full((self.B, max(len(s.block_table) for s in self.seqs)), -1, np.int32)
        for i, s in enumerate(self.seqs):
            self.block_tables[i, :len(s.block_table)] = s.block_table
        md = prepare_prefill(self.seqs, bs)
        if md.total_q != sum(self.lens):
            raise RuntimeError("unexpected prefix-cache hit in a decode workload")
        self.slots_all = md.slot_mapping                 # slot of every position
        cu = np.concatenate([[0], np.cumsum(self.lens)])
        self.last_rows = cu[1:] - 1                      # the decode token of each sequence
        self.decode_slots = self.slots_all[self.last_rows].copy()
        self.max_context_len = max(self.lens)
        self.k = [synth.bf16_normal((L, hkv, d), seed * 31 + 2 * i + 1) for i, L in enumerate(self.lens)]
        self.v = [synth.bf16_normal((L, hkv, d), seed * 31 + 2 * i + 2) for i, L in enumerate(self.lens)]
        self.q = synth.bf16_normal((self.B, hq, d), seed * 31 + 7)

    @classmethod
    def from_spec(cls, w: synth.Workload, block_size=None, **kw):
        lens = list(w.fixed_lens) if w.fixed_lens else \
            synth.uniform_lengths(w.num_seqs, w.ctx_lo, w.ctx_hi, w.seed).tolist()
        return cls(lens, w.num_q_heads, w.num_kv_heads, w.head_dim, block_size or w.block_size,
                   num_blocks=w.num_blocks or None, seed=w.seed, pool_factor=w.pool_factor, **kw)

    # ------------------------------------------------------------------ device
    def upload(self, device="cuda", poison=True):
        """Allocate NaN-poisoned pools, store every prompt row, stage the step's inputs."""
        from . import ops
        shape = (self.nb, self.bs, self.hkv, self.d)
        self.kc = _nan_pool(shape, device) if poison else torch.zeros(shape, dtype=torch.bfloat16, device=device)
        self.vc = self.kc.clone()
        keep = np.ones(sum(self.lens), dtype=bool)
        keep[self.last_rows] = False
        idx = torch.from_numpy(np.nonzero(keep)[0])
        kall, vall = torch.cat(self.k), torch.cat(self.v)
        if len(idx):
            ops.store_kvcache(kall[idx].to(device), vall[idx].to(device), self.kc, self.vc,
                              torch.from_numpy(self.slots_all[keep]).to(device))
        last = torch.from_numpy(self.last_rows)
        self.new_k = kall[last].contiguous()             # host copies (for the e2e path)
        self.new_v = vall[last].contiguous()
        self.d_new_k = self.new_k.to(device)
        self.d_new_v = self.new_v.to(device)
        self.d_q = self.q.to(device)
        self.d_slots = torch.from_numpy(self.decode_slots).to(device)
        self.d_bt = torch.from_numpy(self.block_tables).to(device)
        self.d_cl = torch.tensor(self.lens, dtype=torch.int32, device=device)
        self.d_out = torch.empty((self.B, self.hq, self.d), dtype=torch.bfloat16, device=device)
        self.partition = 0
        from .ops import decode_workspace_size
        ws = decode_workspace_size(self.B, self.hq, self.hkv, self.d, self.max_context_len, 0)
        self.d_ws = torch.empty(max(ws, 1), dtype=torch.uint8, device=device)
        return self

    def step(self, err_flag=None, partition_size=0):
        """One decode step of the hot path: store the new token's K/V, then attend."""
        from . import ops
        ops.store_kvcache(self.d_new_k, self.d_new_v, self.kc, self.vc, self.d_slots, err_flag)
        ws = self.d_ws
        if partition_size:
            need = ops.decode_workspace_size(self.B, self.hq, self.hkv, self.d, self.max_context_len,
                                             partition_size)
            if need > ws.numel():
                ws = torch.empty(need, dtype=torch.uint8, device=self.d_out.device)
        ops.decode(self.d_q, self.kc, self.vc, self.d_bt, self.d_cl, self.max_context_len,
                   out=self.d_out, workspace=ws, partition_size=partition_size, err_flag=err_flag)
        return self.d_out

    # -------------------------------------------------------------- accounting
    def kv_bytes(self) -> int:
        """Algorithmic bytes of one decode launch: every context row's K and V once."""
        return sum(self.lens) * self.hkv * self.d * 2 * 2

    def step_bytes(self) -> int:
        """Decode KV bytes + q read + out write + the store's read and write of the new rows."""
        qo = self.B * self.hq * self.d * 2 * 2
        store = self.B * self.hkv * self.d * 2 * 2 * 2
        return self.kv_bytes() + qo + store


class PrefixPrefillWorkload:
    """Varlen causal prefill where half the sequences share a cached prefix."""

    def __init__(self, hq=28, hkv=4, d=128, bs=256, num_seqs=16, lo=256, hi=2048, prefix=1024,
                 num_shared=8, seed=1004, num_blocks=None):
        self.hq, self.hkv, self.d, self.bs = hq, hkv, d, bs
        rng_lens = synth.uniform_lengths(num_seqs - num_shared, lo, hi, seed)
        shared_lens = synth.uniform_lengths(num_shared, prefix + 1, hi, seed + 1)
        prefix_ids = synth.token_ids(prefix, seed + 2)
        self.prefix = prefix
        # warm-up sequence that holds the prefix blocks (prefilled in an earlier step)
        self.warm = Sequence(prefix_ids + synth.token_ids(1, seed + 3))
        seqs = []
        for i, L in enumerate(rng_lens):
            seqs.append(Sequence(synth.token_ids(int(L), seed + 10 + i)))
        for i, L in enumerate(shared_lens):
            seqs.append(Sequence(prefix_ids + synth.token_ids(int(L) - prefix, seed + 100 + i)))
        self.seqs = seqs
        need = sum(s.num_blocks(bs) for s in seqs) + self.warm.num_blocks(bs)
        self.nb = num_blocks or int(math.ceil(1.25 * need))
        self.bm = BlockManager(self.nb, bs, seed=seed)
        self.bm.allocate(self.warm)
        for s in seqs:
            self.bm.allocate(s)
        self.md = prepare_prefill(seqs, bs)
        self.k_lens = [len(s) for s in seqs]
        self.q_lens = list(np.diff(self.md.cu_seqlens_q))
        self.cached = [s.num_cached_tokens for s in seqs]
        # K/V draws: the warm-up sequence's prefix rows are shared by the prefix-hit sequences
        wl = len(self.warm)
        self.warm_k = synth.bf16_normal((wl, hkv, d), seed * 31 + 1)
        self.warm_v = synth.bf16_normal((wl, hkv, d), seed * 31 + 2)
        self.k, self.v = [], []
        for i, s in enumerate(seqs):
            k = synth.bf16_normal((len(s), hkv, d), seed * 31 + 10 + 2 * i)
            v = synth.bf16_normal((len(s), hkv, d), seed * 31 + 11 + 2 * i)
            c = s.num_cached_tokens
            if c:
                k[:c] = self.warm_k[:c]
                v[:c] = self.warm_v[:c]
            self.k.append(k)
            self.v.append(v)
        self.q = synth.bf16_normal((self.md.total_q, hq, d), seed * 31 + 5)

    def upload(self, device="cuda"):
        from . import ops
        self.kc = _nan_pool((self.nb, self.bs, self.hkv, self.d), device)
        self.vc = self.kc.clone()
        wl = len(self.warm)
        ws = slots_for(self.warm.block_table, 0, wl, self.bs)
        ops.store_kvcache(self.warm_k.to(device), self.warm_v.to(device), self.kc, self.vc,
                          torch.from_numpy(ws).to(device))
        new_k = torch.cat([k[c:] for k, c in zip(self.k, self.cached)])
        new_v = torch.cat([v[c:] for v, c in zip(self.v, self.cached)])
        self.new_k, self.new_v = new_k, new_v
        self.d_new_k, self.d_new_v = new_k.to(device), new_v.to(device)
        self.d_slots = torch.from_numpy(self.md.slot_mapping).to(device)
        self.d_q = self.q.to(device)
        self.d_cu_q = torch.from_numpy(self.md.cu_seqlens_q).to(device)
        self.d_cu_k = torch.from_numpy(self.md.cu_seqlens_k).to(device)
        self.d_bt = torch.from_numpy(self.md.block_tables).to(device)
        self.d_out = torch.empty((self.md.total_q, self.hq, self.d), dtype=torch.bfloat16, device=device)
        return self

    def store(self, err_flag=None):
        from . import ops
        ops.store_kvcache(self.d_new_k, self.d_new_v, self.kc, self.vc, self.d_slots, err_flag)

    def attend(self, err_flag=None):
        from . import ops
        return ops.prefill_varlen(self.d_q, self.kc, self.vc, self.d_cu_q, self.d_cu_k,
                                  self.md.max_seqlen_q, self.md.max_seqlen_k, self.d_bt,
                                  out=self.d_out, err_flag=err_flag)

    def step(self, err_flag=None):
        self.store(err_flag)
        return self.attend(err_flag)

    def fused_step(self, err_flag=None):
        """The same step in one launch: the store folded into the prefill (``prefill_store``)."""
        from . import ops
        return ops.prefill_store(self.d_q, self.d_new_k, self.d_new_v, self.kc, self.vc,
                                 self.d_slots, self.d_cu_q, self.d_cu_k, self.md.max_seqlen_q,
                                 self.md.max_seqlen_k, self.d_bt, out=self.d_out, err_flag=err_flag)

    def flops(self) -> int:
        """Causal algorithmic FLOPs: 4*D*Hq per visible (query, key) pair."""
        total = 0
        for q, c in zip(self.q_lens, self.cached):
            q, c = int(q), int(c)
            total += q * c + q * (q + 1) // 2
        return 4 * self.d * self.hq * total

    def store_bytes(self) -> int:
        return int(self.md.total_q) * self.hkv * self.d * 2 * 2 * 2
