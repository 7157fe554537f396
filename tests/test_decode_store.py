"""pa_decode_store (store + decode in one launch) against the two-launch step (``-m gpu``).

The fused call must leave the pools bit-identical to ``store_kvcache`` and give
bit-identical outputs to ``decode`` (the same kernel arithmetic reads the same
bytes), so the decode's oracle parity carries over; one case is also checked
against the oracle directly.  Edge cases: GQA groups above 16 heads (two CTAs
per KV head both write the new row), split-K partitions, head_dim 64, block 16,
skipped slots (-1), out-of-range slots and slots that break the decode-step
invariant (flags only: the result is then unspecified).
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_attention_35_b200 import synth
from paged_kv_attention_35_b200.workloads import DecodeWorkload
from tests.gpu_cases import DecodeCase, compare
from tests.problems import to_bits

pytestmark = pytest.mark.gpu


def _pair(lens, hq, hkv, d, bs, seed):
    a = DecodeWorkload(lens, hq, hkv, d, bs, seed=seed).upload("cuda")
    b = DecodeWorkload(lens, hq, hkv, d, bs, seed=seed).upload("cuda")
    return a, b


def _fused(ops, w, partition=0, err=None, slots=None):
    ws = w.d_ws
    need = ops.decode_workspace_size(w.B, w.hq, w.hkv, w.d, w.max_context_len, partition)
    if need > ws.numel():
        ws = torch.empty(need, dtype=torch.uint8, device="cuda")
    return ops.decode_store(w.d_q, w.d_new_k, w.d_new_v, w.kc, w.vc,
                            w.d_slots if slots is None else slots, w.d_bt, w.d_cl,
                            w.max_context_len, out=torch.empty_like(w.d_out), workspace=ws,
                            partition_size=partition, err_flag=err)


def _same_pools(a, b):
    assert torch.equal(a.kc.view(torch.int16), b.kc.view(torch.int16))
    assert torch.equal(a.vc.view(torch.int16), b.vc.view(torch.int16))


@pytest.mark.parametrize("hq,hkv,d,bs,partition", [
    (16, 8, 128, 256, 0),      # Qwen3-0.6B shape, automatic split-K
    (16, 8, 128, 256, 128),    # many partitions
    (28, 4, 128, 16, 0),       # GQA 7, block 16
    (40, 2, 128, 64, 256),     # group 20: two q tiles (CTAs) per KV head write the same row
    (8, 2, 64, 32, 64),        # head_dim 64
])
def test_fused_equals_store_then_decode(cuda_device, hq, hkv, d, bs, partition):
    from paged_kv_attention_35_b200 import ops
    lens = [1, 2, 63, 64, 65, 255, 256, 257, 700, 1500, 4000]
    a, b = _pair(lens, hq, hkv, d, bs, seed=900 + hq + bs)
    ref = a.step(partition_size=partition).clone()
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fused(ops, b, partition, err)
    torch.cuda.synchronize()
    _same_pools(a, b)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert int(err.item()) == 0


def test_fused_against_oracle(cuda_device):
    """The tiny decode case through pa_decode_store, checked against the oracle."""
    c = DecodeCase([17, 64, 100, 255], hq=4, hkv=2, d=64, bs=16, num_blocks=64, seed=1001)
    out = c.run_gpu(fused=True)
    kp, vp = c.oracle_pool()
    assert np.array_equal(to_bits(c.kc.cpu()), kp)           # the fused store: bit-exact
    assert np.array_equal(to_bits(c.vc.cpu()), vp)
    compare(out, c.oracle_decode(), "fused tiny decode")


def test_fused_qwen_workload(cuda_device):
    from paged_kv_attention_35_b200 import ops
    spec = synth.WORKLOADS["qwen3_0p6b_decode"]
    a = DecodeWorkload.from_spec(spec).upload("cuda")
    b = DecodeWorkload.from_spec(spec).upload("cuda")
    ref = a.step().clone()
    got = _fused(ops, b)
    torch.cuda.synchronize()
    _same_pools(a, b)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))


def test_fused_skipped_and_bad_slots(cuda_device):
    from paged_kv_attention_35_b200 import ops
    lens = [10, 300, 64]
    a, b = _pair(lens, 8, 2, 128, 16, seed=77)
    # slot -1 for sequence 1: not stored, and attention sees the pool as it is
    slots = a.d_slots.clone()
    slots[1] = -1
    ops.store_kvcache(a.d_new_k, a.d_new_v, a.kc, a.vc, slots)
    ref = ops.decode(a.d_q, a.kc, a.vc, a.d_bt, a.d_cl, a.max_context_len)
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = _fused(ops, b, err=err, slots=slots.clone())
    torch.cuda.synchronize()
    _same_pools(a, b)
    assert torch.equal(got.view(torch.int16), ref.view(torch.int16))
    assert int(err.item()) == 0
    # out of range: skipped with PA_FLAG_SLOT_OOB
    err.zero_()
    bad = b.d_slots.clone()
    bad[0] = b.nb * b.bs + 5
    _fused(ops, b, err=err, slots=bad)
    torch.cuda.synchronize()
    assert int(err.item()) & ops.FLAG_SLOT_OOB
    # in range but not the newest position's slot: PA_FLAG_SLOT_MISMATCH
    err.zero_()
    bad = b.d_slots.clone()
    bad[2] = int(b.d_slots[2].item()) - 1
    _fused(ops, b, err=err, slots=bad)
    torch.cuda.synchronize()
    assert int(err.item()) & ops.FLAG_SLOT_MISMATCH


@pytest.mark.parametrize("name,bs", [
    ("qwen3_0p6b_decode", None),   # config 2: 32 seqs, ctx U[128,4096], 16/8, block 256
    ("gqa7b_decode", 256),         # config 3: 256 seqs, ctx U[512,4096], 28/4, block 256
    ("gqa7b_decode", 16),          # config 3 with 16-token blocks
])
def test_full_size_step_against_oracle(cuda_device, name, bs):
    """The bench's decode step at full size (fused store + decode, automatic partition):
    every sequence's output against the oracle, and the whole pool after the step
    bit-exact against the oracle's own store of every row (prompt rows and the new
    token's) into a NaN-poisoned pool."""
    spec = synth.WORKLOADS[name]
    c = DecodeCase.from_spec(spec, block_size=bs)
    out = c.run_gpu(fused=True)
    compare(out, c.oracle_decode(), f"{name} bs{c.bs}")
    kp, vp = c.oracle_pool()
    assert np.array_equal(to_bits(c.kc.cpu()), kp)
    del kp
    assert np.array_equal(to_bits(c.vc.cpu()), vp)


def test_long_context_decode_against_oracle(cuda_device):
    """Contexts beyond 4096 tokens (16k at block 16, many partitions), GQA 7."""
    c = DecodeCase([16384, 9001, 4097, 300], hq=28, hkv=4, d=128, bs=16, seed=1616)
    out = c.run_gpu(fused=True)
    compare(out, c.oracle_decode(), "long-context decode")
