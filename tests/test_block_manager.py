"""Host control plane: BlockManager, Scheduler and metadata preparation (CPU).

The pages' behavioural rules are the specification here:
prefill-first scheduling, preemption to the head of the waiting queue, block
sharing by hash with reference counts, fixed block size, blocks not cleared
on free, exactly one prefill per sequence (re-prefill only after preemption).
"""

from __future__ import annotations

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

import oracle
from paged_kv_attention_35_b200 import synth
from paged_kv_attention_35_b200.host import (
    BlockManager, PoolExhausted, Scheduler, SchedulerConfig, Sequence, SequenceStatus,
    PriorityScheduler, prepare_decode, prepare_prefill,
)


def test_allocate_pops_seeded_permutation_in_order():
    bm = BlockManager(64, 16, seed=1001)
    order = np.random.default_rng(1001).permutation(64).tolist()
    a = Sequence(list(range(17)))
    b = Sequence(list(range(100, 164)))
    bm.allocate(a)
    bm.allocate(b)
    assert a.block_table == order[:2]
    assert b.block_table == order[2:6]
    bm.check_invariants([a, b])


def test_free_appends_right_and_keeps_hash():
    bm = BlockManager(8, 4)
    s = Sequence([1, 2, 3, 4, 5, 6, 7, 8, 9])
    bm.allocate(s)
    ids = list(s.block_table)
    bm.deallocate(s)
    assert list(bm.free_block_ids)[-3:] == ids[::-1]
    # hashed full blocks survive on the free list and are revived by a hit
    t = Sequence([1, 2, 3, 4, 5, 6, 7, 8, 42, 43])
    bm.allocate(t)
    assert t.block_table[:2] == ids[:2]
    assert t.num_cached_tokens == 8
    bm.check_invariants([t])


def test_prefix_hit_shares_blocks_with_ref_count():
    bm = BlockManager(32, 4, seed=3)
    prefix = [7] * 4 + [8] * 4 + [9] * 4
    a = Sequence(prefix + [1, 2])
    b = Sequence(prefix + [3])
    bm.allocate(a)
    bm.allocate(b)
    assert b.block_table[:3] == a.block_table[:3]
    assert b.num_cached_tokens == 12
    for bid in a.block_table[:3]:
        assert bm.blocks[bid].ref_count == 2
    assert b.block_table[3] != a.block_table[3]
    bm.check_invariants([a, b])
    bm.deallocate(a)
    for bid in b.block_table[:3]:
        assert bm.blocks[bid].ref_count == 1
    bm.check_invariants([b])


def test_hash_is_chained_and_needs_equal_tokens():
    bm = BlockManager(32, 4)
    a = Sequence([1, 1, 1, 1, 2, 2, 2, 2, 5])
    bm.allocate(a)
    # same second block, different first block: chained hash misses on block 2 too
    b = Sequence([9, 9, 9, 9, 2, 2, 2, 2, 5])
    bm.allocate(b)
    assert b.num_cached_tokens == 0
    assert set(a.block_table).isdisjoint(b.block_table)


def test_last_token_block_is_always_computed():
    bm = BlockManager(16, 4)
    a = Sequence(list(range(8)))
    bm.allocate(a)
    b = Sequence(list(range(8)))               # identical, prompt a multiple of the block size
    bm.allocate(b)
    assert b.num_cached_tokens == 4            # the block holding the last token is recomputed
    assert b.block_table[0] == a.block_table[0] and b.block_table[1] != a.block_table[1]
    md = prepare_prefill([b], 4)
    assert md.total_q == 4


def test_collision_guard():
    bm = BlockManager(16, 4)
    a = Sequence([1, 2, 3, 4, 5])
    bm.allocate(a)
    h = bm.blocks[a.block_table[0]].hash
    bm.blocks[a.block_table[0]].token_ids = [0, 0, 0, 0]      # pretend a colliding entry
    b = Sequence([1, 2, 3, 4, 6])
    bm.allocate(b)
    assert b.num_cached_tokens == 0
    assert h == bm.blocks[a.block_table[0]].hash


def test_append_slot_adds_block_and_hashes_full_block():
    bs = 4
    bm = BlockManager(8, bs)
    s = Sequence([1, 2, 3])
    bm.allocate(s)
    s.append_token(4)                          # position 3 fills block 0
    assert not bm.needs_new_block(s)
    bm.append_slot(s)
    assert bm.blocks[s.block_table[0]].hash != -1
    s.append_token(5)                          # position 4 starts block 1
    assert bm.needs_new_block(s)
    bm.append_slot(s)
    assert len(s.block_table) == 2
    bm.check_invariants([s])
    # a later sequence with the same first block hits it
    t = Sequence([1, 2, 3, 4, 9])
    bm.allocate(t)
    assert t.block_table[0] == s.block_table[0]


def test_slot_mapping_matches_oracle():
    bs = 16
    bm = BlockManager(64, bs, seed=1001)
    seqs = [Sequence(synth.token_ids(L, 5 + L)) for L in (17, 64, 100, 255)]
    for s in seqs:
        bm.allocate(s)
    md = prepare_prefill(seqs, bs)
    for i, s in enumerate(seqs):
        a, b = md.cu_seqlens_q[i], md.cu_seqlens_q[i + 1]
        ref = oracle.ref_slot_mapping(s.block_table, range(s.num_cached_tokens, len(s)), bs)
        assert np.array_equal(md.slot_mapping[a:b], ref)
    for s in seqs:
        s.append_token(1)
        bm.append_slot(s)
    dm = prepare_decode(seqs, bs)
    for i, s in enumerate(seqs):
        assert dm.context_lens[i] == len(s)
        assert dm.slot_mapping[i] == oracle.ref_slot_mapping(s.block_table, [len(s) - 1], bs)[0]
    assert dm.block_tables.dtype == np.int32 and (dm.block_tables[0, 2:] == -1).all()


def _cfg(**kw):
    base = dict(max_num_seqs=4, max_num_batched_tokens=64, block_size=4, num_blocks=16, seed=0)
    base.update(kw)
    return SchedulerConfig(**base)


def test_prefill_first_then_decode():
    sch = Scheduler(_cfg())
    a = Sequence([1] * 5, max_tokens=3)
    sch.add(a)
    seqs, is_prefill = sch.schedule()
    assert is_prefill and seqs == [a]
    sch.postprocess(seqs, [2])
    b = Sequence([3] * 6, max_tokens=2)
    sch.add(b)
    seqs, is_prefill = sch.schedule()            # waiting non-empty -> prefill first
    assert is_prefill and seqs == [b]
    sch.postprocess(seqs, [4])
    seqs, is_prefill = sch.schedule()
    assert not is_prefill and seqs == [a, b]


def test_token_budget_and_max_num_seqs():
    sch = Scheduler(_cfg(max_num_batched_tokens=10, num_blocks=64, max_num_seqs=2))
    seqs = [Sequence([i] * 6, max_tokens=1) for i in range(3)]
    for s in seqs:
        sch.add(s)
    batch, _ = sch.schedule()
    assert batch == seqs[:1]                     # 6 + 6 > 10
    batch, _ = sch.schedule()
    assert batch == seqs[1:2]                    # max_num_seqs = 2 running
    assert len(sch.waiting) == 1


def test_preemption_to_head_of_waiting():
    # 4 blocks of 4 tokens; two sequences of 7 tokens use 2 blocks each, decode needs a 3rd
    sch = Scheduler(_cfg(num_blocks=4, max_num_seqs=4))
    a = Sequence([1] * 7, max_tokens=5)
    b = Sequence([2] * 7, max_tokens=5)
    sch.add(a); sch.add(b)
    batch, pf = sch.schedule()
    assert pf and batch == [a, b]
    sch.postprocess(batch, [0, 0])               # both now 8 tokens: fit exactly
    batch, pf = sch.schedule()
    assert not pf and batch == [a, b]
    sch.postprocess(batch, [0, 0])               # 9 tokens: each needs a new block, none free
    batch, pf = sch.schedule()
    assert not pf and batch == [a]               # newest (b) preempted
    assert sch.waiting[0] is b and b.status == SequenceStatus.WAITING
    assert b.block_table == [] and sch.num_preemptions == 1
    sch.block_manager.check_invariants([a])


def test_self_preemption_when_last_in_batch():
    # a and b hold 2 blocks each of a 4-block pool; b reaches a block boundary first and,
    # with nobody behind it to evict, preempts itself
    sch = Scheduler(_cfg(num_blocks=4, max_num_seqs=4))
    a = Sequence([1] * 6, max_tokens=4)
    b = Sequence([2] * 7, max_tokens=4)
    sch.add(a); sch.add(b)
    batch, _ = sch.schedule()
    sch.postprocess(batch, [0, 0])                # a: 7, b: 8 tokens
    batch, pf = sch.schedule()
    assert not pf and batch == [a, b]
    sch.postprocess(batch, [0, 0])                # a: 8, b: 9 -> b needs a 5th block
    batch, pf = sch.schedule()
    assert batch == [a] and list(sch.waiting) == [b] and b.num_preemptions == 1


def test_sequence_too_long_is_rejected():
    sch = Scheduler(_cfg(num_blocks=2))
    with pytest.raises(ValueError):
        sch.add(Sequence([1] * 9, max_tokens=4))


def test_priority_scheduler_admits_highest_first():
    sch = PriorityScheduler(_cfg(max_num_seqs=1, num_blocks=64))
    lo = Sequence([1] * 3, priority=0)
    hi = Sequence([2] * 3, priority=5)
    sch.add(lo); sch.add(hi)
    batch, pf = sch.schedule()
    assert pf and batch == [hi]


def _run_trace(num_req, seed, num_blocks, bs, max_num_seqs, budget, check_every=1):
    rng = np.random.default_rng(seed)
    sch = Scheduler(SchedulerConfig(max_num_seqs=max_num_seqs, max_num_batched_tokens=budget,
                                    block_size=bs, num_blocks=num_blocks, seed=seed))
    prefix = rng.integers(0, 50, size=2 * bs).tolist()
    reqs = []
    for r in range(num_req):
        n = int(rng.integers(1, 3 * bs))
        toks = (prefix if r % 2 else []) + rng.integers(0, 50, size=n).tolist()
        s = Sequence(toks, max_tokens=int(rng.integers(1, 2 * bs)))
        reqs.append(s)
        sch.add(s)
    steps = prefills = 0
    seen_prefill = {}
    while not sch.is_finished():
        batch, pf = sch.schedule()
        assert batch
        steps += 1
        live = list(sch.running)
        if steps % check_every == 0:
            sch.block_manager.check_invariants(live)
        if pf:
            prefills += 1
            for s in batch:
                # one prefill per sequence unless it was preempted in between
                seen_prefill[s.seq_id] = seen_prefill.get(s.seq_id, 0) + 1
                assert seen_prefill[s.seq_id] == 1 + s.num_preemptions
            md = prepare_prefill(batch, bs)
            assert md.total_q >= len(batch)
        else:
            md = prepare_decode(batch, bs)
            # every slot of the step is distinct and owned by its sequence
            assert len(set(md.slot_mapping.tolist())) == len(batch)
        sch.postprocess(batch, rng.integers(0, 50, size=len(batch)).tolist())
    assert all(s.is_finished for s in reqs)
    assert all(s.num_completion_tokens == s.max_tokens for s in reqs)
    bm = sch.block_manager
    assert bm.num_free_blocks == num_blocks
    return steps, sch.num_preemptions, bm.prefix_hit_tokens


def test_trace_runs_to_completion_with_preemption_and_hits():
    steps, pre, hits = _run_trace(40, 7, num_blocks=24, bs=4, max_num_seqs=8, budget=64)
    assert pre > 0 and hits > 0


def test_trace_is_deterministic():
    assert _run_trace(20, 9, 24, 4, 6, 48) == _run_trace(20, 9, 24, 4, 6, 48)


@settings(max_examples=25, deadline=None)
@given(seed=st.integers(0, 10_000), nb=st.integers(12, 40), bs=st.sampled_from([2, 4, 8]),
       mns=st.integers(1, 8))
def test_trace_property(seed, nb, bs, mns):
    # the pool must hold the longest single request (3*bs prompt + 2*bs prefix + 2*bs output)
    nb = max(nb, 8)
    _run_trace(12, seed, nb, bs, mns, budget=8 * bs)
