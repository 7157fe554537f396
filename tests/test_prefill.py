"""GPU parity of varlen causal prefill (with cached prefixes) against the oracle."""

from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_attention_35_b200 import synth
from tests.gpu_cases import (PrefillCase, PrefixPrefillWorkload, compare, oracle_prefix_prefill,
                             rows_of)

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("bs", [16, 64, 256])
@pytest.mark.parametrize("hq,hkv,d", [(28, 4, 128), (16, 8, 128), (8, 1, 64)])
def test_prefill_ragged(cuda_device, bs, hq, hkv, d):
    # (cached, new): no cache, cache not block aligned, one new token, tile edges
    cached = [0, 0, 0, 17, 256, 300, 0, 5, 1024]
    new = [1, 63, 129, 47, 1, 200, 256, 64, 65]
    c = PrefillCase(cached, new, hq=hq, hkv=hkv, d=d, bs=bs, seed=11 + bs + hq)
    out = c.run_gpu()
    compare(out, c.oracle_prefill(), f"prefill bs{bs} {hq}/{hkv} d{d}")


def test_prefill_long_uncached(cuda_device):
    c = PrefillCase([0, 0], [2048, 777], hq=28, hkv=4, d=128, bs=256, seed=3)
    compare(c.run_gpu(), c.oracle_prefill(), "long")


def test_prefix_cached_prefill_workload(cuda_device):
    """16 seqs, 8 fresh U[256,2048], 8 sharing a 1024-token hash-cached prefix;
    28/4 heads, D 128, block 256.  Every sequence checked against the oracle."""
    w = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4).upload("cuda")
    assert sum(1 for c in w.cached if c == 1024) == 8          # the 8 prefix hits
    out = w.step().clone()
    torch.cuda.synchronize()
    compare(out, oracle_prefix_prefill(w), "prefix prefill")


def test_shared_prefix_equals_private_copy(cuda_device):
    """Sequences reading hash-shared prefix blocks give bit-identical outputs to
    the same sequences reading private copies of those blocks."""
    w = PrefixPrefillWorkload(num_seqs=4, num_shared=2, lo=300, hi=1500, seed=21).upload("cuda")
    shared = w.step().clone()
    bt = w.d_bt.clone()
    nb = w.nb
    extra = 0
    kc = torch.cat([w.kc, torch.empty_like(w.kc[:8])])
    vc = torch.cat([w.vc, torch.empty_like(w.vc[:8])])
    for i, c in enumerate(w.cached):
        for j in range(c // w.bs):
            src = int(bt[i, j])
            dst = nb + extra
            extra += 1
            kc[dst] = kc[src]
            vc[dst] = vc[src]
            bt[i, j] = dst
    assert extra > 0
    from paged_kv_attention_35_b200 import ops
    private = ops.prefill_varlen(w.d_q, kc, vc, w.d_cu_q, w.d_cu_k, w.md.max_seqlen_q,
                                 w.md.max_seqlen_k, bt)
    torch.cuda.synchronize()
    assert torch.equal(shared, private)


def test_decode_matches_last_prefill_row(cuda_device):
    """Decode at context L == the last row of an uncached prefill of length L (same q)."""
    from paged_kv_attention_35_b200 import ops
    L = 777
    c = PrefillCase([0], [L], hq=16, hkv=8, d=128, bs=16, seed=5)
    pre = c.run_gpu()
    bt = torch.from_numpy(c.block_tables).cuda()
    q_last = c.q[L - 1:L].cuda()
    dec = ops.decode(q_last, c.kc, c.vc, bt, torch.tensor([L], dtype=torch.int32, device="cuda"), L)
    torch.cuda.synchronize()
    diff = (dec[0].float() - pre[L - 1].float()).abs()
    assert diff.max() <= 2e-2


def test_first_row_of_uncached_prefill_is_v0(cuda_device):
    c = PrefillCase([0, 0], [40, 300], hq=8, hkv=2, d=128, bs=64, seed=6)
    out = c.run_gpu().cpu()
    for i in range(2):
        r = int(c.cu_q[i])
        for h in range(8):
            assert torch.equal(out[r, h], c.v[i][0, h // 4])


def test_prefill_checked_mode(cuda_device):
    c = PrefillCase([0, 20], [50, 30], hq=4, hkv=2, d=128, bs=16, seed=7)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    c.run_gpu(err_flag=flag)
    assert int(flag.item()) == 0
    from paged_kv_attention_35_b200 import ops
    bt = torch.from_numpy(c.block_tables).cuda()
    bt[1, 0] = -5
    out = ops.prefill_varlen(c.q.cuda(), c.kc, c.vc, torch.from_numpy(c.cu_q).cuda(),
                             torch.from_numpy(c.cu_k).cuda(), 50, 50, bt, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & ops.FLAG_BLOCK_OOB
    assert torch.isfinite(out.float()).all()
    flag.zero_()
    cu_k = torch.from_numpy(c.cu_k).cuda()
    cu_k[2] = cu_k[1] + 10                     # k_len < q_len: inconsistent
    ops.prefill_varlen(c.q.cuda(), c.kc, c.vc, torch.from_numpy(c.cu_q).cuda(), cu_k, 50, 50,
                       torch.from_numpy(c.block_tables).cuda(), err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & ops.FLAG_LEN_OOB


@pytest.mark.parametrize("hq,hkv,d", [(12, 4, 128), (40, 2, 128), (8, 8, 128), (14, 2, 64)])
def test_prefill_group_packing(cuda_device, hq, hkv, d):
    """Query tiles pack floor(128 / G) queries x the G heads of a KV head as MMA rows:
    groups of 3 (126 rows), 20 (120 rows), 1 (128 rows) and 7 at head_dim 64, with
    ragged lengths, cached prefixes and a sequence with no new query."""
    cached = [0, 5, 300, 0, 1000, 17]
    new = [1, 50, 0, 257, 40, 700]
    c = PrefillCase(cached, new, hq=hq, hkv=hkv, d=d, bs=64, seed=40 + hq + d)
    out = c.run_gpu()
    compare(out, c.oracle_prefill(), f"prefill {hq}/{hkv} d{d}")


@pytest.mark.parametrize("d", [64, 128])
def test_prefill_largest_group(cuda_device, d):
    """128 query heads on one KV head, the most a tile packs: one query per tile, so
    every pair of queries is a unit."""
    c = PrefillCase([0, 5, 130], [3, 40, 17], hq=128, hkv=1, d=d, bs=16, seed=61 + d)
    compare(c.run_gpu(), c.oracle_prefill(), f"prefill group 128 d{d}")


def test_prefill_many_sequences(cuda_device):
    """More work units than SMs: each persistent CTA walks many units."""
    rng = np.random.default_rng(99)
    new = rng.integers(1, 200, size=300).tolist()
    cached = rng.integers(0, 300, size=300).tolist()
    c = PrefillCase(cached, new, hq=16, hkv=8, d=128, bs=16, seed=12)
    out = c.run_gpu()
    seqs = list(range(0, 300, 7))
    compare(out[torch.from_numpy(c.rows_of(seqs)).cuda()], c.oracle_prefill(seqs), "many seqs")


def test_prefill_block_table_past_staged_entries(cuda_device):
    """Block 16 with 5,000-token sequences: a unit's keys span up to 313 blocks, past the 256
    block-table entries the producer stages in shared memory (the rest are read directly)."""
    c = PrefillCase([1000, 3], [4000, 4997], hq=8, hkv=2, d=64, bs=16, seed=41)
    compare(c.run_gpu(), c.oracle_prefill(), "prefill past staged block-table entries")


@pytest.mark.parametrize("hq,hkv,d", [(28, 4, 128), (8, 1, 64)])
def test_prefill_output_only_16_byte_aligned(cuda_device, hq, hkv, d):
    """An output buffer that is 16- but not 32-byte aligned takes the 16-byte store path of
    the epilogue (32-byte stores otherwise): the same bits either way."""
    from paged_kv_attention_35_b200 import ops
    c = PrefillCase([0, 17, 300], [129, 47, 200], hq=hq, hkv=hkv, d=d, bs=64, seed=5 + d)
    ref = c.run_gpu()
    assert ref.data_ptr() % 32 == 0
    buf = torch.zeros(ref.numel() + 8, dtype=torch.bfloat16, device=ref.device)
    out = buf[8:].view(ref.shape)
    assert out.data_ptr() % 32 == 16
    ops.prefill_varlen(c.q.to(ref.device), c.kc, c.vc, torch.from_numpy(c.cu_q).to(ref.device),
                       torch.from_numpy(c.cu_k).to(ref.device), max(c.new), max(c.k_lens),
                       torch.from_numpy(c.block_tables).to(ref.device), out=out)
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    assert torch.equal(buf[:8].view(torch.int16), torch.zeros(8, dtype=torch.int16, device=ref.device))
