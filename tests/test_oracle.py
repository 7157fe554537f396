"""Pins for the CPU oracle (no GPU).

Each check ties the oracle to something other than itself: the scalar brute
force, a library routine (torch's float64 scaled-dot-product attention on the
CPU, on K/V that never went through the oracle's gather), closed forms, the
worked examples in ``tests/golden/``, and invariants.  ``test_planted_*``
plants plausible mistakes in the oracle (on the CPU) and shows that the
checks catch each one.
"""

from __future__ import annotations

import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
import oracle.paged as op
from oracle import brute
from tests.problems import decode_problem, prefill_problem, to_bits, from_bits, build_pool

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
f64 = oracle.bf16_bits_to_f64


def _sdpa(q, k, v, causal=False, scale=None):
    """torch float64 SDPA on the CPU: q [Lq, D], k/v [Lk, D] -> [Lq, D]."""
    qt = torch.from_numpy(q)[None, None]
    kt = torch.from_numpy(k)[None, None]
    vt = torch.from_numpy(v)[None, None]
    o = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, is_causal=causal, scale=scale)
    return o[0, 0].numpy()


# ----------------------------------------------------------------- the checks
# Written as plain functions so the planted-mistake tests can rerun them.

def check_bf16_conversion():
    allbits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = f64(allbits)
    lib = from_bits(allbits).to(torch.float64).numpy()
    same = (ours == lib) | (np.isnan(ours) & np.isnan(lib))
    assert same.all()
    # rounding: float32 values (exact in float64) against torch's float32 -> bf16 cast
    x = torch.randn(200000, generator=torch.Generator().manual_seed(3)) * 10.0
    x = torch.cat([x, torch.tensor([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -(1.0 + 2 ** -8), 3e38, 1e-40])])
    ours = oracle.f64_to_bf16_bits(x.double().numpy())
    lib = to_bits(x.to(torch.bfloat16))
    assert (ours == lib).all()


def check_decode_brute():
    p = decode_problem([1, 5, 16, 37], hq=4, hkv=2, d=8, bs=4, seed=11)
    q = f64(p["q"])
    kp, vp = f64(p["k_pool"]), f64(p["v_pool"])
    got = oracle.ref_decode(q, kp, vp, p["block_tables"], p["lens"])
    ref = np.asarray(brute.brute_decode(q, kp, vp, p["block_tables"], p["lens"]))
    assert np.abs(got - ref).max() <= 1e-12


def check_prefill_brute():
    p = prefill_problem([3, 40, 1], [3, 45, 20], hq=6, hkv=2, d=8, bs=4, seed=12)
    q = f64(p["q"])
    kp, vp = f64(p["k_pool"]), f64(p["v_pool"])
    got = oracle.ref_prefill(q, kp, vp, p["cu_q"], p["cu_k"], p["block_tables"])
    ref = np.asarray(brute.brute_prefill(q, kp, vp, p["cu_q"], p["cu_k"], p["block_tables"]))
    assert np.abs(got - ref).max() <= 1e-12


def check_decode_library():
    """Paged decode == torch SDPA on the logical (never paged) K/V."""
    p = decode_problem([17, 64, 100, 255], hq=4, hkv=2, d=64, bs=16, num_blocks=64, seed=21)
    q = f64(p["q"])
    got = oracle.ref_decode(q, f64(p["k_pool"]), f64(p["v_pool"]), p["block_tables"], p["lens"])
    for i in range(4):
        K, V = f64(p["k_logical"][i]), f64(p["v_logical"][i])
        for h in range(4):
            ref = _sdpa(q[i, h][None], K[:, h // 2], V[:, h // 2])[0]
            assert np.abs(got[i, h] - ref).max() <= 1e-12


def check_prefill_library():
    """Uncached prefill == torch SDPA with is_causal on the logical K/V."""
    p = prefill_problem([33, 70], [33, 70], hq=4, hkv=1, d=16, bs=8, seed=22)
    q = f64(p["q"])
    got = oracle.ref_prefill(q, f64(p["k_pool"]), f64(p["v_pool"]), p["cu_q"], p["cu_k"],
                             p["block_tables"])
    for i in range(2):
        a, b = p["cu_q"][i], p["cu_q"][i + 1]
        K, V = f64(p["k_logical"][i]), f64(p["v_logical"][i])
        for h in range(4):
            ref = _sdpa(q[a:b, h], K[:, 0], V[:, 0], causal=True)
            assert np.abs(got[a:b, h] - ref).max() <= 1e-12


def check_cached_prefix_is_suffix():
    """A prefill with c cached tokens == the last rows of the uncached prefill."""
    c, n = 23, 31
    p = prefill_problem([c + n], [c + n], hq=2, hkv=2, d=8, bs=8, seed=23)
    q = f64(p["q"])
    kp, vp = f64(p["k_pool"]), f64(p["v_pool"])
    full = oracle.ref_prefill(q, kp, vp, p["cu_q"], p["cu_k"], p["block_tables"])
    tail = oracle.ref_prefill(q[c:], kp, vp, np.array([0, n]), p["cu_k"], p["block_tables"])
    assert np.abs(full[c:] - tail).max() <= 1e-12


def check_decode_is_last_prefill_row():
    """Decode at context L == last row of an uncached prefill of length L."""
    L = 29
    p = prefill_problem([L], [L], hq=4, hkv=2, d=8, bs=4, seed=24)
    q = f64(p["q"])
    kp, vp = f64(p["k_pool"]), f64(p["v_pool"])
    pre = oracle.ref_prefill(q, kp, vp, p["cu_q"], p["cu_k"], p["block_tables"])
    dec = oracle.ref_decode(q[L - 1:L], kp, vp, p["block_tables"], np.array([L]))
    assert np.abs(pre[L - 1] - dec[0]).max() <= 1e-12


def check_closed_forms():
    rng = np.random.default_rng(5)
    d, hkv, hq, bs, L = 8, 2, 4, 4, 13
    # (i) equal keys -> mean of V over attended rows (decode: all L; prefill row j: k_len-q_len+j+1)
    krow = rng.standard_normal((1, hkv, d))
    kl = np.repeat(krow, L, axis=0)
    vl = rng.standard_normal((L, hkv, d))
    bt = np.array([[5, 0, 3, 1]], dtype=np.int32)
    kp = np.zeros((6, bs, hkv, d)); vp = np.zeros((6, bs, hkv, d))
    for j in range(4):
        kp[bt[0, j], :len(kl[j * bs:(j + 1) * bs])] = kl[j * bs:(j + 1) * bs]
        vp[bt[0, j], :len(vl[j * bs:(j + 1) * bs])] = vl[j * bs:(j + 1) * bs]
    q = rng.standard_normal((1, hq, d))
    out = oracle.ref_decode(q, kp, vp, bt, [L])
    for h in range(hq):
        assert np.abs(out[0, h] - vl[:, h // 2].mean(axis=0)).max() <= 1e-12
    qp = rng.standard_normal((5, hq, d))
    outp = oracle.ref_prefill(qp, kp, vp, [0, 5], [0, L], bt)
    for j in range(5):
        n_att = L - 5 + j + 1
        for h in range(hq):
            assert np.abs(outp[j, h] - vl[:n_att, h // 2].mean(axis=0)).max() <= 1e-12
    # (ii) a single attended key -> that V row exactly
    out1 = oracle.ref_decode(q, kp, vp, bt, [1])
    for h in range(hq):
        assert np.array_equal(out1[0, h], vl[0, h // 2])
    # (iii) one key whose score beats the rest by > 50 -> its V row
    k3 = rng.standard_normal((L, hkv, d)) * 0.01
    k3[7] = 0.0
    qd = np.zeros((1, hq, d)); qd[0, :, 0] = 1.0
    k3[7, :, 0] = 60.0 * math.sqrt(d)
    kp3 = kp.copy()
    for j in range(4):
        kp3[bt[0, j], :len(k3[j * bs:(j + 1) * bs])] = k3[j * bs:(j + 1) * bs]
    out3 = oracle.ref_decode(qd, kp3, vp, bt, [L])
    for h in range(hq):
        assert np.abs(out3[0, h] - vl[7, h // 2]).max() <= 1e-12
    # (iv) identical q across a GQA group -> identical outputs inside the group
    qg = rng.standard_normal((1, hq, d))
    qg[0, 1] = qg[0, 0]
    qg[0, 3] = qg[0, 2]
    og = oracle.ref_decode(qg, kp, vp, bt, [L])
    assert np.array_equal(og[0, 0], og[0, 1]) and np.array_equal(og[0, 2], og[0, 3])
    assert not np.allclose(og[0, 0], og[0, 2])


def _expected(case):
    """The fixture's expected values are closed-form expressions in e = exp(1)."""
    env = {"__builtins__": {}, "e": math.e, "exp": math.exp}
    return np.asarray([[eval(x, env) for x in row] if isinstance(row, list) else eval(row, env)
                       for row in case["expected"]], dtype=float)


def check_worked_examples():
    """Hand-derived examples in tests/golden/worked_examples.json."""
    with open(os.path.join(GOLDEN, "worked_examples.json")) as f:
        ex = json.load(f)
    for case in ex["decode"]:
        k = np.asarray(case["keys"], float)[:, None, :]        # [L, 1, D]
        v = np.asarray(case["values"], float)[:, None, :]
        L, _, d = k.shape
        kp = k[None]; vp = v[None]                             # one block of size L
        out = oracle.ref_decode(np.asarray(case["q"], float)[None, None], kp, vp,
                                np.array([[0]]), [L], scale=case["scale"])
        assert np.abs(out[0, 0] - _expected(case)).max() <= 1e-12, case["name"]
    for case in ex["prefill"]:
        k = np.asarray(case["keys"], float)[:, None, :]
        v = np.asarray(case["values"], float)[:, None, :]
        q = np.asarray(case["queries"], float)[:, None, :]
        kp = k[None]; vp = v[None]
        out = oracle.ref_prefill(q, kp, vp, [0, q.shape[0]], [0, k.shape[0]], np.array([[0]]),
                                 scale=case["scale"])
        assert np.abs(out[:, 0] - _expected(case)).max() <= 1e-12, case["name"]


def check_layout_invariance():
    """Block sizes 4 / 16 / one whole block, and permuted block ids: same result."""
    lens = [5, 31, 64]
    outs = []
    for bs, seed_perm in [(4, 1), (16, 2), (64, 3), (4, 9)]:
        p = decode_problem(lens, hq=4, hkv=2, d=8, bs=bs, seed=31)   # same logical draws
        # re-place the same logical rows under a different block permutation
        from tests.problems import assign_blocks
        nb = p["num_blocks"]
        bt = assign_blocks(lens, bs, nb, seed_perm)
        kp = build_pool(p["k_logical"], bt, bs, nb, 2, 8)
        vp = build_pool(p["v_logical"], bt, bs, nb, 2, 8)
        outs.append(oracle.ref_decode(f64(p["q"]), f64(kp), f64(vp), bt, p["lens"]))
    for o in outs[1:]:
        assert np.array_equal(o, outs[0])
    for o in outs:
        assert np.isfinite(o).all()


def check_gather_roundtrip():
    p = decode_problem([3, 17, 40], hq=2, hkv=2, d=8, bs=8, seed=41)
    for i in range(3):
        g = oracle.ref_gather(p["k_pool"], p["block_tables"][i], int(p["lens"][i]))
        assert np.array_equal(g, p["k_logical"][i])


def check_slot_mapping():
    bs = 16
    bt = np.array([9, 2, 7, 0], dtype=np.int32)
    pos = np.arange(0, 61)
    slots = oracle.ref_slot_mapping(bt, pos, bs)
    # enumerate the pool block by block: logical block j row r is slot bt[j]*bs + r
    expect = []
    for j in range(4):
        for r in range(bs):
            expect.append(bt[j] * bs + r)
    assert np.array_equal(slots, np.asarray(expect[:61]))
    assert len(set(slots.tolist())) == 61


def check_store():
    rng = np.random.default_rng(7)
    nb, bs, hkv, d = 6, 4, 2, 8
    kp = rng.integers(0, 65535, (nb, bs, hkv, d)).astype(np.uint16)
    vp = rng.integers(0, 65535, (nb, bs, hkv, d)).astype(np.uint16)
    key = rng.integers(0, 65535, (5, hkv, d)).astype(np.uint16)
    val = rng.integers(0, 65535, (5, hkv, d)).astype(np.uint16)
    slots = np.array([3, -1, 22, 0, 9])
    k2, v2 = oracle.ref_store(kp, vp, key, val, slots)
    for i, s in enumerate(slots):
        if s < 0:
            continue
        assert np.array_equal(k2[s // bs, s % bs], key[i])
        assert np.array_equal(v2[s // bs, s % bs], val[i])
    touched = {int(s) for s in slots if s >= 0}
    for s in range(nb * bs):
        if s not in touched:
            assert np.array_equal(k2[s // bs, s % bs], kp[s // bs, s % bs])
            assert np.array_equal(v2[s // bs, s % bs], vp[s // bs, s % bs])
    assert np.array_equal(kp, kp.copy())          # inputs untouched


def check_prefill_flops():
    cu_q = [0, 5, 12, 13]
    cu_k = [0, 5, 20, 43]
    q = np.diff(cu_q); k = np.diff(cu_k); c = k - q
    closed = 4 * 16 * 3 * int(np.sum(q * c + q * (q + 1) // 2))
    assert oracle.ref_prefill_flops(cu_q, cu_k, 3, 16) == closed


ALL_CHECKS = [check_bf16_conversion, check_decode_brute, check_prefill_brute, check_decode_library,
              check_prefill_library, check_cached_prefix_is_suffix, check_decode_is_last_prefill_row,
              check_closed_forms, check_worked_examples, check_layout_invariance,
              check_gather_roundtrip, check_slot_mapping, check_store, check_prefill_flops]


@pytest.mark.parametrize("check", ALL_CHECKS, ids=lambda f: f.__name__)
def test_oracle_pin(check):
    check()


# ------------------------------------------------------------ planted mistakes

def _fails(checks):
    """True when at least one check rejects the (mutated) oracle.

    A crash (e.g. an index that leaves the pool) counts as a rejection too.
    """
    for c in checks:
        try:
            c()
        except Exception:
            return True
    return False


ATTN_CHECKS = [check_decode_brute, check_prefill_brute, check_decode_library,
               check_prefill_library, check_cached_prefix_is_suffix,
               check_decode_is_last_prefill_row, check_closed_forms, check_worked_examples]


@pytest.mark.parametrize("name,target,mutant", [
    ("gqa head modulo", "_kv_head", lambda h, g: h % 2),
    ("gqa group boundary shifted", "_kv_head", lambda h, g: (h + 1) // g),
    ("causal off by one (sees next key)", "_last_visible_key", lambda kl, ql, j: kl - ql + j + 1),
    ("causal misses diagonal", "_last_visible_key", lambda kl, ql, j: max(kl - ql + j - 1, 0)),
    ("top-left causal alignment", "_last_visible_key", lambda kl, ql, j: j),
    ("no softmax scale", "_default_scale", lambda d: 1.0),
    ("scale 1/d", "_default_scale", lambda d: 1.0 / d),
])
def test_planted_attention_mistake(monkeypatch, name, target, mutant):
    monkeypatch.setattr(op, target, mutant)
    # the brute force and library checks do not go through the patched helper,
    # so at least one of them must now disagree
    assert _fails(ATTN_CHECKS), name


def test_planted_softmax_mistake(monkeypatch):
    def no_max_sub_wrong_norm(s, v):
        p = np.exp(s)
        return (p / (p.sum() + 1.0)) @ v          # a dropped/extra term in the normaliser
    monkeypatch.setattr(op, "_softmax_attend", no_max_sub_wrong_norm)
    assert _fails(ATTN_CHECKS)


def test_planted_gather_mistake(monkeypatch):
    real = op.ref_gather

    def reversed_blocks(pool, block_table, length):
        bs = pool.shape[1]
        n = -(-length // bs)
        return real(pool, list(block_table[:n])[::-1], length)
    monkeypatch.setattr(op, "ref_gather", reversed_blocks)
    assert _fails(ATTN_CHECKS + [check_gather_roundtrip])


def test_planted_store_mistake(monkeypatch):
    real = op.ref_store

    def store_ignores_skip(kp, vp, key, val, slots):
        return real(kp, vp, key, val, np.abs(np.asarray(slots)))
    monkeypatch.setattr(oracle, "ref_store", store_ignores_skip)
    assert _fails([check_store])


def test_planted_slot_mistake(monkeypatch):
    def transposed(bt, positions, bs):
        return np.asarray([int(bt[p % len(bt)]) * bs + p // len(bt) for p in positions])
    monkeypatch.setattr(oracle, "ref_slot_mapping", transposed)
    assert _fails([check_slot_mapping])


def test_planted_bf16_mistake(monkeypatch):
    def truncating(x):
        f32 = np.asarray(x, np.float64).astype(np.float32)
        return (f32.view(np.uint32) >> np.uint32(16)).astype(np.uint16)
    monkeypatch.setattr(oracle, "f64_to_bf16_bits", truncating)
    assert _fails([check_bf16_conversion])
