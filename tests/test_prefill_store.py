"""GPU parity of the fused prefill store (``pa_prefill_store``): one launch that
writes the step's new K/V rows to the pool and runs the causal varlen prefill.

The bar is bit-identity with the two-launch step it replaces -- ``store_kvcache``
of the new rows, then ``prefill_varlen`` -- on both the output and the whole pool
(NaN-filled beforehand, so a stray or missing write shows), plus the oracle on
the output.  Cases cover cached lengths that are and are not multiples of the
TMA box (a box holding cached and new keys is read from the pool after its new
rows are written), block sizes 16 / 64 / 256, the head shapes of the prefill
tests, strided key/value (slices of one packed qkv buffer), tokens past the last
sequence, and the slot checks.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from paged_kv_attention_35_b200 import synth
from paged_kv_attention_35_b200.host.prepare import slots_for
from tests.gpu_cases import PrefillCase, PrefixPrefillWorkload, compare, oracle_prefix_prefill

pytestmark = pytest.mark.gpu


def _bits(t: torch.Tensor) -> torch.Tensor:
    return t.view(torch.int16)


def _prefix_pools(c: PrefillCase, dev="cuda"):
    """NaN-filled pools holding the case's cached prefixes (an earlier step)."""
    from paged_kv_attention_35_b200 import ops
    kc = torch.full((c.nb, c.bs, c.hkv, c.d), synth.NAN_BF16_BITS, dtype=torch.int16,
                    device=dev).view(torch.bfloat16)
    vc = kc.clone()
    rk, rv, sl = [], [], []
    for i in range(len(c.k_lens)):
        if c.cached[i]:
            rk.append(c.k[i][:c.cached[i]])
            rv.append(c.v[i][:c.cached[i]])
            sl.append(slots_for(c.block_tables[i], 0, c.cached[i], c.bs))
    if rk:
        ops.store_kvcache(torch.cat(rk).to(dev), torch.cat(rv).to(dev), kc, vc,
                          torch.from_numpy(np.concatenate(sl)).to(dev))
    return kc, vc


def _new_rows(c: PrefillCase, dev="cuda"):
    """This step's new K/V rows in packed token order and their slots."""
    k = torch.cat([c.k[i][c.cached[i]:] for i in range(len(c.k_lens))]).to(dev)
    v = torch.cat([c.v[i][c.cached[i]:] for i in range(len(c.k_lens))]).to(dev)
    s = np.concatenate([slots_for(c.block_tables[i], c.cached[i], c.k_lens[i], c.bs)
                        for i in range(len(c.k_lens))]).astype(np.int32)
    return k, v, torch.from_numpy(s).to(dev)


def _two_launch(c, key, value, slots, q, cu_q, cu_k, bt, stored=None):
    """Reference step: store_kvcache of the first `stored` tokens, then prefill_varlen."""
    from paged_kv_attention_35_b200 import ops
    kc, vc = _prefix_pools(c)
    n = key.shape[0] if stored is None else stored
    ops.store_kvcache(key[:n], value[:n], kc, vc, slots[:n])
    out = ops.prefill_varlen(q, kc, vc, cu_q, cu_k, max(c.new), max(c.k_lens), bt)
    torch.cuda.synchronize()
    return out, kc, vc


def _fused(c, key, value, slots, q, cu_q, cu_k, bt):
    from paged_kv_attention_35_b200 import ops
    kc, vc = _prefix_pools(c)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    out = ops.prefill_store(q, key, value, kc, vc, slots, cu_q, cu_k, max(c.new), max(c.k_lens),
                            bt, err_flag=flag)
    torch.cuda.synchronize()
    return out, kc, vc, int(flag.item())


def _inputs(c):
    q = c.q.to("cuda")
    cu_q = torch.from_numpy(c.cu_q).cuda()
    cu_k = torch.from_numpy(c.cu_k).cuda()
    bt = torch.from_numpy(c.block_tables).cuda()
    return q, cu_q, cu_k, bt


def _check_same(a, b, what):
    out_a, kc_a, vc_a = a[:3]
    out_b, kc_b, vc_b = b[:3]
    assert torch.equal(_bits(out_a), _bits(out_b)), f"{what}: output differs"
    assert torch.equal(_bits(kc_a), _bits(kc_b)), f"{what}: K pool differs"
    assert torch.equal(_bits(vc_a), _bits(vc_b)), f"{what}: V pool differs"


@pytest.mark.parametrize("bs", [16, 64, 256])
@pytest.mark.parametrize("hq,hkv,d", [(28, 4, 128), (16, 8, 128), (8, 1, 64)])
def test_fused_equals_store_then_prefill(cuda_device, bs, hq, hkv, d):
    # cached lengths 17, 300, 5 are not multiples of any box (16, 64, 128 rows)
    cached = [0, 0, 0, 17, 256, 300, 0, 5, 1024]
    new = [1, 63, 129, 47, 1, 200, 256, 64, 65]
    c = PrefillCase(cached, new, hq=hq, hkv=hkv, d=d, bs=bs, seed=11 + bs + hq)
    key, value, slots = _new_rows(c)
    q, cu_q, cu_k, bt = _inputs(c)
    ref = _two_launch(c, key, value, slots, q, cu_q, cu_k, bt)
    got = _fused(c, key, value, slots, q, cu_q, cu_k, bt)
    assert got[3] == 0, f"err_flag {got[3]}"
    _check_same(got, ref, f"bs{bs} {hq}/{hkv} d{d}")
    compare(got[0], c.oracle_prefill(), f"fused prefill bs{bs} {hq}/{hkv} d{d}")


@pytest.mark.parametrize("hq,hkv,d,bs", [(14, 2, 64, 16), (40, 2, 128, 64), (12, 4, 128, 256)])
def test_fused_group_packing_and_empty_sequences(cuda_device, hq, hkv, d, bs):
    """Groups of 7, 20 and 3 query heads per KV head, a sequence with no new
    tokens (nothing to store), one new token after a long unaligned prefix."""
    c = PrefillCase([0, 40, 0, 999, 3], [30, 0, 1, 1, 250], hq=hq, hkv=hkv, d=d, bs=bs, seed=7 + hq)
    key, value, slots = _new_rows(c)
    q, cu_q, cu_k, bt = _inputs(c)
    ref = _two_launch(c, key, value, slots, q, cu_q, cu_k, bt)
    got = _fused(c, key, value, slots, q, cu_q, cu_k, bt)
    assert got[3] == 0
    _check_same(got, ref, f"group {hq // hkv}")
    compare(got[0], c.oracle_prefill(), f"fused group {hq // hkv}")


def test_fused_prefix_prefill_workload(cuda_device):
    """The prefix-cached prefill workload (16 sequences, 8 of them sharing a
    1024-token hash-cached prefix; 28/4 heads, D 128, block 256) in one launch:
    pools and output bit-identical to store-then-prefill, every sequence
    against the oracle."""
    two = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4).upload("cuda")
    ref = two.step().clone()
    one = PrefixPrefillWorkload(seed=synth.SEED_BASE + 4).upload("cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    got = one.fused_step(err_flag=flag).clone()
    torch.cuda.synchronize()
    assert int(flag.item()) == 0
    assert torch.equal(_bits(got), _bits(ref))
    assert torch.equal(_bits(one.kc), _bits(two.kc))
    assert torch.equal(_bits(one.vc), _bits(two.vc))
    compare(got, oracle_prefix_prefill(one), "fused prefix prefill")


def test_fused_strided_qkv(cuda_device):
    """q, key and value as column slices of one packed [T, (Hq + 2 Hkv) D] buffer."""
    hq, hkv, d = 28, 4, 128
    c = PrefillCase([0, 130, 512], [300, 77, 129], hq=hq, hkv=hkv, d=d, bs=64, seed=19)
    key, value, slots = _new_rows(c)
    T = key.shape[0]
    qkv = torch.empty((T, (hq + 2 * hkv) * d), dtype=torch.bfloat16, device="cuda")
    qkv[:, :hq * d] = c.q.to("cuda").reshape(T, -1)
    qkv[:, hq * d:(hq + hkv) * d] = key.reshape(T, -1)
    qkv[:, (hq + hkv) * d:] = value.reshape(T, -1)
    q = qkv[:, :hq * d].view(T, hq, d)
    ks = qkv[:, hq * d:(hq + hkv) * d].view(T, hkv, d)
    vs = qkv[:, (hq + hkv) * d:].view(T, hkv, d)
    assert ks.stride(0) == (hq + 2 * hkv) * d
    _, cu_q, cu_k, bt = _inputs(c)
    ref = _two_launch(c, ks, vs, slots, q, cu_q, cu_k, bt)
    got = _fused(c, ks, vs, slots, q, cu_q, cu_k, bt)
    assert got[3] == 0
    _check_same(got, ref, "strided qkv")


def test_fused_tokens_past_last_sequence(cuda_device):
    """Rows past cu_seqlens_q[num_seqs] belong to no sequence: not stored, not computed."""
    c = PrefillCase([0, 200], [150, 90], hq=16, hkv=8, d=128, bs=16, seed=23)
    key, value, slots = _new_rows(c)
    n, pad = key.shape[0], 9
    key = torch.cat([key, key[:pad]])
    value = torch.cat([value, value[:pad]])
    # valid-looking slots: the first rows of blocks no sequence uses
    used = set(int(b) for b in c.block_tables.ravel() if b >= 0)
    free = [b for b in range(c.nb) if b not in used]
    assert free
    slots = torch.cat([slots, torch.arange(pad, dtype=torch.int32, device="cuda") + free[0] * c.bs])
    q, cu_q, cu_k, bt = _inputs(c)
    q = torch.cat([q, q[:pad]])
    ref = _two_launch(c, key, value, slots, q, cu_q, cu_k, bt, stored=n)
    got = _fused(c, key, value, slots, q, cu_q, cu_k, bt)
    assert got[3] == 0
    assert torch.equal(_bits(got[0][:n]), _bits(ref[0][:n]))
    assert torch.equal(_bits(got[1]), _bits(ref[1])) and torch.equal(_bits(got[2]), _bits(ref[2]))


def test_fused_slot_checks(cuda_device):
    """A slot that is not its position's block-table slot raises PA_FLAG_SLOT_MISMATCH;
    one past the pool raises PA_FLAG_SLOT_OOB and writes nothing."""
    from paged_kv_attention_35_b200 import ops
    c = PrefillCase([0, 64], [100, 40], hq=16, hkv=8, d=128, bs=16, seed=29)
    key, value, slots = _new_rows(c)
    q, cu_q, cu_k, bt = _inputs(c)
    swapped = slots.clone()
    swapped[[3, 4]] = swapped[[4, 3]]
    got = _fused(c, key, value, swapped, q, cu_q, cu_k, bt)
    assert got[3] & ops.FLAG_SLOT_MISMATCH and not got[3] & ops.FLAG_SLOT_OOB
    oob = slots.clone()
    oob[120] = c.nb * c.bs
    got = _fused(c, key, value, oob, q, cu_q, cu_k, bt)
    assert got[3] & ops.FLAG_SLOT_OOB
    # every other row is in place, the out-of-pool row went nowhere
    ref = _two_launch(c, key, value, oob, q, cu_q, cu_k, bt)
    assert torch.equal(_bits(got[1]), _bits(ref[1])) and torch.equal(_bits(got[2]), _bits(ref[2]))


def test_fused_block_table_past_staged_entries(cuda_device):
    """The fused store at block 16 with 5,000-token sequences (block tables longer than the
    256 entries staged per unit; a cached length of 3 leaves a box of cached and new keys)."""
    c = PrefillCase([1000, 3], [4000, 4997], hq=8, hkv=2, d=64, bs=16, seed=43)
    key, value, slots = _new_rows(c)
    q, cu_q, cu_k, bt = _inputs(c)
    ref = _two_launch(c, key, value, slots, q, cu_q, cu_k, bt)
    got = _fused(c, key, value, slots, q, cu_q, cu_k, bt)
    assert got[3] == 0
    _check_same(got, ref, "block 16, 5000 tokens")


def test_fused_random_configs(cuda_device):
    """Twelve seeded random batches: block size 16..1024, head shapes with groups of 1 to 16,
    D 64 or 128, 1-6 sequences with cached lengths 0..700 (aligned to the box or not) and
    1..400 new tokens; output and pools bit-identical to store-then-prefill, no flags."""
    import random
    rnd = random.Random(2024)
    shapes = [(8, 8, 64), (16, 8, 128), (28, 4, 128), (32, 2, 64), (16, 1, 128), (12, 3, 128)]
    for case in range(12):
        hq, hkv, d = rnd.choice(shapes)
        bs = rnd.choice([16, 32, 64, 128, 256, 1024])
        nseq = rnd.randint(1, 6)
        cached = [rnd.choice([0, 0, rnd.randint(1, 700), 128 * rnd.randint(1, 5)]) for _ in range(nseq)]
        new = [rnd.randint(1, 400) for _ in range(nseq)]
        c = PrefillCase(cached, new, hq=hq, hkv=hkv, d=d, bs=bs, seed=300 + case)
        key, value, slots = _new_rows(c)
        q, cu_q, cu_k, bt = _inputs(c)
        ref = _two_launch(c, key, value, slots, q, cu_q, cu_k, bt)
        got = _fused(c, key, value, slots, q, cu_q, cu_k, bt)
        assert got[3] == 0, (case, got[3])
        _check_same(got, ref, f"random case {case}: {hq}/{hkv} d{d} bs{bs} {cached} {new}")
