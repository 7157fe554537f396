"""End-to-end GPU cases built through the product's control plane and kernels,
with the oracle's expectation computed independently on the CPU.

Flow of a decode case (``DecodeWorkload``): the product's ``BlockManager``
places each sequence's tokens (seeded shuffled pool), ``prepare_prefill``
gives the slots of every position and the last position is the decode
token's; the GPU pool starts NaN-poisoned, ``store_kvcache`` writes the prompt
rows, then a step stores the new token's rows and runs ``decode``.  The oracle recomputes every
slot from the block tables (``ref_slot_mapping``), applies ``ref_store`` to its
own NaN pool and runs ``ref_decode`` on the result; nothing it uses comes from
the GPU.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from paged_kv_attention_35_b200 import synth
from paged_kv_attention_35_b200.workloads import DecodeWorkload, PrefixPrefillWorkload
from tests.problems import to_bits, from_bits, build_pool

TOL_MAX = 2e-2
TOL_MEAN = 2e-3


def compare(got_bf16: torch.Tensor, ref_f64: np.ndarray, what: str = ""):
    got = got_bf16.float().cpu().double().numpy()
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref_f64)
    mx, mean = float(err.max()), float(err.mean())
    assert mx <= TOL_MAX and mean <= TOL_MEAN, f"{what}: max {mx:.3e} mean {mean:.3e}"
    return mx, mean


def pool_need(lens, bs):
    return sum(-(-int(L) // bs) for L in lens)


class DecodeCase(DecodeWorkload):
    """A decode workload plus the oracle's independent expectation."""

    def run_gpu(self, partition_size=0, err_flag=None, poison=True, fused=False):
        """The decode step on the GPU: store_kvcache then decode, or (``fused``) both
        through pa_decode_store in one launch.  Also keeps the output as ``self.out``."""
        self.upload(poison=poison)
        if fused:
            from paged_kv_attention_35_b200 import ops
            ws = self.d_ws
            need = ops.decode_workspace_size(self.B, self.hq, self.hkv, self.d,
                                             self.max_context_len, partition_size)
            if need > ws.numel():
                ws = torch.empty(need, dtype=torch.uint8, device=self.d_out.device)
            out = ops.decode_store(self.d_q, self.d_new_k, self.d_new_v, self.kc, self.vc,
                                   self.d_slots, self.d_bt, self.d_cl, self.max_context_len,
                                   out=self.d_out, workspace=ws, partition_size=partition_size,
                                   err_flag=err_flag).clone()
        else:
            out = self.step(err_flag=err_flag, partition_size=partition_size).clone()
        torch.cuda.synchronize()
        self.bt_dev, self.cl_dev = self.d_bt, self.d_cl
        self.out = out
        return out

    # ------------------------------------------------------------ oracle side
    def oracle_slots(self):
        out = []
        for i, L in enumerate(self.lens):
            out.append(oracle.ref_slot_mapping(self.block_tables[i], range(L), self.bs))
        return np.concatenate(out)

    def oracle_pool(self):
        kp = np.full((self.nb, self.bs, self.hkv, self.d), synth.NAN_BF16_BITS, np.uint16)
        vp = kp.copy()
        kp, vp = oracle.ref_store(kp, vp, to_bits(torch.cat(self.k)), to_bits(torch.cat(self.v)),
                                  self.oracle_slots())
        return kp, vp

    def oracle_decode(self, rows=None):
        """Expected output for sequences `rows` (all when None), float64."""
        rows = list(range(len(self.lens))) if rows is None else list(rows)
        sub_lens = [self.lens[i] for i in rows]
        # a compact pool holding only these sequences' rows (renumbered blocks)
        bt = np.full((len(rows), self.block_tables.shape[1]), -1, np.int32)
        k = 0
        for j, L in enumerate(sub_lens):
            n = -(-L // self.bs)
            bt[j, :n] = np.arange(k, k + n)
            k += n
        kp = build_pool([to_bits(self.k[i]) for i in rows], bt, self.bs, max(k, 1), self.hkv, self.d)
        vp = build_pool([to_bits(self.v[i]) for i in rows], bt, self.bs, max(k, 1), self.hkv, self.d)
        q = oracle.bf16_bits_to_f64(to_bits(self.q))[rows]
        return oracle.ref_decode(q, oracle.bf16_bits_to_f64(kp), oracle.bf16_bits_to_f64(vp), bt,
                                 np.asarray(sub_lens))


class PrefillCase:
    """Sequences with ``cached`` prefix tokens already in the pool and ``new`` tokens to compute."""

    def __init__(self, cached, new, hq, hkv, d, bs, num_blocks=None, seed=0, device="cuda",
                 share_prefix=None):
        self.cached = [int(c) for c in cached]
        self.new = [int(n) for n in new]
        self.k_lens = [c + n for c, n in zip(self.cached, self.new)]
        self.hq, self.hkv, self.d, self.bs = hq, hkv, d, bs
        need = pool_need(self.k_lens, bs)
        self.nb = num_blocks or max(need + 1, int(math.ceil(1.25 * need)))
        bt = np.full((len(self.k_lens), max(-(-L // bs) for L in self.k_lens)), -1, np.int32)
        order = synth.permutation(self.nb, seed + 3).tolist()
        k = 0
        for i, L in enumerate(self.k_lens):
            n = -(-L // bs)
            bt[i, :n] = order[k:k + n]
            k += n
        self.block_tables = bt
        self.k = [synth.bf16_normal((L, hkv, d), seed * 31 + 2 * i + 1) for i, L in enumerate(self.k_lens)]
        self.v = [synth.bf16_normal((L, hkv, d), seed * 31 + 2 * i + 2) for i, L in enumerate(self.k_lens)]
        self.q = synth.bf16_normal((sum(self.new), hq, d), seed * 31 + 5)
        self.cu_q = np.concatenate([[0], np.cumsum(self.new)]).astype(np.int32)
        self.cu_k = np.concatenate([[0], np.cumsum(self.k_lens)]).astype(np.int32)
        self.device = device

    def run_gpu(self, err_flag=None):
        from paged_kv_attention_35_b200 import ops
        from paged_kv_attention_35_b200.host import slots_for
        dev = self.device
        kc = torch.full((self.nb, self.bs, self.hkv, self.d), synth.NAN_BF16_BITS, dtype=torch.int16,
                        device=dev).view(torch.bfloat16)
        vc = kc.clone()
        # cached prefix rows (an earlier step), then the new rows (this step)
        for part in ("cached", "new"):
            rows_k, rows_v, slots = [], [], []
            for i in range(len(self.k_lens)):
                a, b = (0, self.cached[i]) if part == "cached" else (self.cached[i], self.k_lens[i])
                if b > a:
                    rows_k.append(self.k[i][a:b])
                    rows_v.append(self.v[i][a:b])
                    slots.append(slots_for(self.block_tables[i], a, b, self.bs))
            if rows_k:
                ops.store_kvcache(torch.cat(rows_k).to(dev), torch.cat(rows_v).to(dev), kc, vc,
                                  torch.from_numpy(np.concatenate(slots)).to(dev), err_flag)
        self.kc, self.vc = kc, vc
        out = ops.prefill_varlen(self.q.to(dev), kc, vc, torch.from_numpy(self.cu_q).to(dev),
                                 torch.from_numpy(self.cu_k).to(dev), max(self.new), max(self.k_lens),
                                 torch.from_numpy(self.block_tables).to(dev), err_flag=err_flag)
        torch.cuda.synchronize()
        return out

    def oracle_prefill(self, seqs=None):
        """Expected rows of sequences `seqs` (all when None) in packed order, float64."""
        seqs = list(range(len(self.k_lens))) if seqs is None else list(seqs)
        k_lens = [self.k_lens[i] for i in seqs]
        bt = np.full((len(seqs), self.block_tables.shape[1]), -1, np.int32)
        k = 0
        for j, L in enumerate(k_lens):
            n = -(-L // self.bs)
            bt[j, :n] = np.arange(k, k + n)
            k += n
        kp = oracle.bf16_bits_to_f64(build_pool([to_bits(self.k[i]) for i in seqs], bt, self.bs,
                                                max(k, 1), self.hkv, self.d))
        vp = oracle.bf16_bits_to_f64(build_pool([to_bits(self.v[i]) for i in seqs], bt, self.bs,
                                                max(k, 1), self.hkv, self.d))
        qall = oracle.bf16_bits_to_f64(to_bits(self.q))
        q = np.concatenate([qall[self.cu_q[i]:self.cu_q[i + 1]] for i in seqs])
        cu_q = np.concatenate([[0], np.cumsum([self.new[i] for i in seqs])])
        cu_k = np.concatenate([[0], np.cumsum(k_lens)])
        return oracle.ref_prefill(q, kp, vp, cu_q, cu_k, bt)

    def rows_of(self, seqs):
        return np.concatenate([np.arange(self.cu_q[i], self.cu_q[i + 1]) for i in seqs])


def oracle_prefix_prefill(w: PrefixPrefillWorkload, seqs=None):
    """Oracle rows for sequences `seqs` of a prefix-cached prefill workload (packed order)."""
    seqs = list(range(len(w.seqs))) if seqs is None else list(seqs)
    k_lens = [w.k_lens[i] for i in seqs]
    bt = np.full((len(seqs), max(-(-L // w.bs) for L in k_lens)), -1, np.int32)
    k = 0
    for j, L in enumerate(k_lens):
        n = -(-L // w.bs)
        bt[j, :n] = np.arange(k, k + n)
        k += n
    kp = oracle.bf16_bits_to_f64(build_pool([to_bits(w.k[i]) for i in seqs], bt, w.bs, k, w.hkv, w.d))
    vp = oracle.bf16_bits_to_f64(build_pool([to_bits(w.v[i]) for i in seqs], bt, w.bs, k, w.hkv, w.d))
    cu = w.md.cu_seqlens_q
    qall = oracle.bf16_bits_to_f64(to_bits(w.q))
    q = np.concatenate([qall[cu[i]:cu[i + 1]] for i in seqs])
    cu_q = np.concatenate([[0], np.cumsum([w.q_lens[i] for i in seqs])])
    cu_k = np.concatenate([[0], np.cumsum(k_lens)])
    return oracle.ref_prefill(q, kp, vp, cu_q, cu_k, bt)


def rows_of(cu_q, seqs):
    return np.concatenate([np.arange(cu_q[i], cu_q[i + 1]) for i in seqs])
