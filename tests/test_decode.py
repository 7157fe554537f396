"""GPU parity of store_kvcache + paged decode against the oracle (``-m gpu``).

Tolerance (attention outputs, bf16 in / fp32 accumulate / bf16 out, against
float64): max abs 2e-2 and mean abs 2e-3; store and all slot / block indexing
are bit-exact.
"""

from __future__ import annotations

import numpy as np
import pytest
import torch

from tests.gpu_cases import DecodeCase, compare
from tests.problems import to_bits

pytestmark = pytest.mark.gpu


def test_tiny_decode_step(cuda_device):
    """4 seqs, context lens [17,64,100,255], 4 Q / 2 KV heads, D 64, block 16, 64-block pool."""
    c = DecodeCase([17, 64, 100, 255], hq=4, hkv=2, d=64, bs=16, num_blocks=64, seed=1001)
    out = c.run_gpu()
    kp, vp = c.oracle_pool()
    assert np.array_equal(to_bits(c.kc.cpu()), kp)           # store: bit-exact, poison intact
    assert np.array_equal(to_bits(c.vc.cpu()), vp)
    assert np.array_equal(c.slots_all, c.oracle_slots())
    compare(out, c.oracle_decode(), "tiny decode")


@pytest.mark.parametrize("bs", [16, 32, 64, 256])
@pytest.mark.parametrize("hq,hkv,d", [(16, 8, 128), (28, 4, 128), (8, 1, 64), (4, 4, 128)])
def test_decode_shapes(cuda_device, bs, hq, hkv, d):
    lens = [1, 2, 15, 16, 17, 63, 64, 65, 127, 129, 300, 511, 777, 1024, 1500]
    c = DecodeCase(lens, hq=hq, hkv=hkv, d=d, bs=bs, seed=7 + bs + hq)
    out = c.run_gpu()
    compare(out, c.oracle_decode(), f"decode bs{bs} {hq}/{hkv} d{d}")


@pytest.mark.parametrize("partition", [64, 128, 256, 512, 0])
def test_split_k_partitions(cuda_device, partition):
    lens = [5, 64, 640, 1000, 2049, 4096]
    c = DecodeCase(lens, hq=28, hkv=4, d=128, bs=256, seed=55)
    out = c.run_gpu(partition_size=partition)
    compare(out, c.oracle_decode(), f"partition {partition}")


def test_large_group_over_16(cuda_device):
    """GQA groups larger than 16 use several query tiles per KV head."""
    c = DecodeCase([33, 400, 1030], hq=40, hkv=2, d=128, bs=16, seed=9)
    compare(c.run_gpu(), c.oracle_decode(), "group 20")


@pytest.mark.parametrize("d", [64, 128])
def test_largest_group(cuda_device, d):
    """128 query heads on one KV head: eight query tiles per KV head."""
    c = DecodeCase([1, 300, 1000], hq=128, hkv=1, d=d, bs=16, seed=13 + d)
    compare(c.run_gpu(), c.oracle_decode(), f"group 128 d{d}")


def test_layout_and_permutation_invariance(cuda_device):
    """Same logical K/V and q under block sizes 16 / 256 / one block per sequence
    and under two shuffles of the pool: each within tolerance of the oracle, and
    bit-identical to one another (the kernel's reduction order follows logical
    positions only)."""
    lens = [100, 700, 1000, 1024]
    outs = []
    for bs, pool_seed in [(16, 1), (256, 1), (1024, 1), (256, 2)]:
        c = DecodeCase(lens, hq=16, hkv=8, d=128, bs=bs, seed=77, pool_seed=pool_seed)
        out = c.run_gpu(partition_size=256)
        compare(out, c.oracle_decode(), f"bs {bs} pool {pool_seed}")
        outs.append(out)
    for o in outs[1:]:
        assert torch.equal(o, outs[0]), "output depends on the physical layout"


def test_single_key_is_exact(cuda_device):
    """context_len 1: the output is the V row itself, bit-exact in bf16."""
    c = DecodeCase([1, 1, 1], hq=8, hkv=2, d=128, bs=16, seed=3)
    out = c.run_gpu().cpu()
    for i in range(3):
        for h in range(8):
            assert torch.equal(out[i, h], c.v[i][0, h // 4])


def test_equal_keys_give_mean_of_v(cuda_device):
    c = DecodeCase([300, 1000], hq=8, hkv=2, d=128, bs=256, seed=4)
    for i in range(2):
        c.k[i][:] = c.k[i][0:1]
    out = c.run_gpu().cpu().double()
    for i in range(2):
        mean = c.v[i].double().mean(dim=0)              # [Hkv, D]
        for h in range(8):
            err = (out[i, h] - mean[h // 4]).abs()
            assert err.max() <= 2e-2 and err.mean() <= 2e-3


def test_identical_queries_in_group(cuda_device):
    c = DecodeCase([90, 513], hq=16, hkv=2, d=128, bs=32, seed=5)
    c.q[:, 1] = c.q[:, 0]
    out = c.run_gpu().cpu()
    assert torch.equal(out[:, 0], out[:, 1])


def test_nan_poisoned_tail_does_not_leak(cuda_device):
    # every pool row outside the contexts is NaN (see DecodeCase.run_gpu)
    c = DecodeCase([3, 17, 250, 257], hq=4, hkv=2, d=64, bs=256, seed=6)
    out = c.run_gpu()
    assert torch.isfinite(out.float()).all()


def test_checked_mode_flags_bad_block_ids(cuda_device):
    c = DecodeCase([40, 80], hq=4, hkv=2, d=64, bs=16, seed=8)
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    c.run_gpu(err_flag=flag)
    assert int(flag.item()) == 0
    from paged_kv_attention_35_b200 import ops
    bt = c.bt_dev.clone()
    bt[1, 2] = c.nb + 100                      # out of range block id
    out = ops.decode(c.q.cuda(), c.kc, c.vc, bt, c.cl_dev, 80, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & ops.FLAG_BLOCK_OOB
    assert torch.isfinite(out.float()).all()  # the bad block reads zeros, nothing faults
    flag.zero_()
    cl = c.cl_dev.clone()
    cl[0] = 0
    out = ops.decode(c.q.cuda(), c.kc, c.vc, c.bt_dev, cl, 80, err_flag=flag)
    torch.cuda.synchronize()
    assert int(flag.item()) & ops.FLAG_LEN_OOB
    assert torch.equal(out[0].float().cpu(), torch.zeros_like(out[0].float().cpu()))
    assert ops.watchdog_read() == 0


def test_store_skips_negative_and_flags_out_of_range(cuda_device):
    from paged_kv_attention_35_b200 import ops
    nb, bs, hkv, d = 8, 16, 2, 64
    kc = torch.zeros(nb, bs, hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    key = torch.randn(4, hkv, d, device="cuda").to(torch.bfloat16)
    val = torch.randn(4, hkv, d, device="cuda").to(torch.bfloat16)
    slots = torch.tensor([5, -1, nb * bs, 127], dtype=torch.int32, device="cuda")
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")
    ops.store_kvcache(key, val, kc, vc, slots, flag)
    torch.cuda.synchronize()
    assert int(flag.item()) == ops.FLAG_SLOT_OOB
    flat = kc.view(nb * bs, hkv, d)
    assert torch.equal(flat[5], key[0]) and torch.equal(flat[127], key[3])
    assert int((flat != 0).any(dim=(1, 2)).sum()) == 2
    assert torch.equal(vc.view(nb * bs, hkv, d)[127], val[3])


def test_store_strided_rows(cuda_device):
    """key/value may be views into a packed QKV projection output (token stride > row)."""
    from paged_kv_attention_35_b200 import ops
    hq, hkv, d, n = 16, 8, 128, 37
    qkv = torch.randn(n, (hq + 2 * hkv) * d, device="cuda").to(torch.bfloat16)
    k = qkv[:, hq * d:(hq + hkv) * d].view(n, hkv, d)
    v = qkv[:, (hq + hkv) * d:].view(n, hkv, d)
    kc = torch.zeros(4, 16, hkv, d, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    slots = torch.randperm(64, device="cuda")[:n].to(torch.int32)
    ops.store_kvcache(k, v, kc, vc, slots)
    torch.cuda.synchronize()
    flat_k = kc.view(64, hkv, d)
    flat_v = vc.view(64, hkv, d)
    assert torch.equal(flat_k[slots.long()], k) and torch.equal(flat_v[slots.long()], v)


def test_empty_batch_is_noop(cuda_device):
    from paged_kv_attention_35_b200 import ops
    kc = torch.zeros(4, 16, 2, 64, dtype=torch.bfloat16, device="cuda")
    e = torch.zeros(0, 2, 64, dtype=torch.bfloat16, device="cuda")
    ops.store_kvcache(e, e, kc, kc.clone(), torch.zeros(0, dtype=torch.int32, device="cuda"))
    q = torch.zeros(0, 4, 64, dtype=torch.bfloat16, device="cuda")
    out = ops.decode(q, kc, kc, torch.zeros(0, 1, dtype=torch.int32, device="cuda"),
                     torch.zeros(0, dtype=torch.int32, device="cuda"), 16)
    assert out.shape == (0, 4, 64)


def test_store_full_size_permutation(cuda_device):
    """The bench's bulk store at full size (65,536 rows, 8 x 128 bf16 each, slots a
    seeded permutation of the whole pool): every pool row equals the input row the
    permutation sends there -- bit-exact, checked through the inverse permutation."""
    from paged_kv_attention_35_b200 import ops, synth
    n, hkv, d, bs = 65536, 8, 128, 256
    key = synth.bf16_normal((n, hkv, d), 7).cuda()
    val = synth.bf16_normal((n, hkv, d), 8).cuda()
    kc = torch.full((n // bs, bs, hkv, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    vc = torch.full_like(kc, float("nan"))
    perm = synth.permutation(n, 9).astype(np.int64)
    ops.store_kvcache(key, val, kc, vc, torch.from_numpy(perm.astype(np.int32)).cuda())
    torch.cuda.synchronize()
    inv = np.empty(n, np.int64)
    inv[perm] = np.arange(n)
    idx = torch.from_numpy(inv).cuda()
    assert torch.equal(kc.view(n, hkv, d).view(torch.int16), key[idx].view(torch.int16))
    assert torch.equal(vc.view(n, hkv, d).view(torch.int16), val[idx].view(torch.int16))


def test_bounded_wait_gives_up_and_reports(cuda_device):
    """Failure detection: a wait nothing completes gives up after its limit, reports
    PA_FLAG_TIMEOUT in err_flag and in the watchdog word, and the context stays
    usable (a decode step right after is checked against the oracle)."""
    from paged_kv_attention_35_b200 import ops
    ops.watchdog_read()                                      # clear
    err = torch.zeros(1, dtype=torch.int32, device="cuda")
    waited = torch.zeros(1, dtype=torch.int64, device="cuda")
    ops.selftest_wait_timeout(50_000, err, waited)
    torch.cuda.synchronize()
    assert int(err.item()) & ops.FLAG_TIMEOUT
    assert 50e6 <= int(waited.item()) < 2e9
    assert ops.watchdog_read() & ops.FLAG_TIMEOUT
    assert ops.watchdog_read() == 0                          # read clears it
    c = DecodeCase([17, 64, 100, 255], hq=4, hkv=2, d=64, bs=16, num_blocks=64, seed=1001)
    compare(c.run_gpu(), c.oracle_decode(), "decode after a timed-out wait")
